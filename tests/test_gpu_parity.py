"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Bar (fixed for every case here):
  - routing indices, expert counts, offsets, padded offsets, gather_idx and inv_pos:
    bit-exact;
  - gate weights: |w_gpu - w_ref| <= 1e-6 * w_ref + 1e-7 (fp32 expf, subtraction, sum and
    division on the GPU against fp64 on the oracle's side; a few fp32 roundings of
    relative size 2^-24 each);
  - layer output (bf16) against the fp64 oracle: |out - ref| <= 2e-2 + 2e-2 * |ref|
    element-wise;
  - combine on given bf16 rows: |out - ref| <= 2^-8 * |ref| + 1e-6 (one bf16 rounding of
    an fp32 sum);
  - two identical calls give bit-identical outputs.
"""
import math

import numpy as np
import pytest
import torch

import mixture_experts_layer_forward_b200 as moe
import oracle
from mixture_experts_layer_forward_b200 import synth

pytestmark = pytest.mark.gpu

ATOL, RTOL = 2e-2, 2e-2
GATE_RTOL, GATE_ATOL = 1e-6, 1e-7


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    torch.cuda.set_device(0)
    moe.library()


def bits(t):
    return synth.bf16_bits(t)


def alloc_ws(p):
    n = moe.moe_workspace_size(p)
    assert n > 0
    return torch.empty(n, dtype=torch.uint8, device="cuda")


def cfg_small(name, T, H, F, E, k, **kw):
    return synth.LayerConfig(name, T=T, H=H, F=F, E=E, k=k, **kw)


def run_forward(cfg, inp, ws=None):
    p = moe.Problem.from_config(cfg)
    ws = alloc_ws(p) if ws is None else ws
    d = {k: (v.cuda() if v is not None else None) for k, v in inp.items()}
    out = torch.empty(cfg.T, cfg.H, dtype=torch.bfloat16, device="cuda")
    idx = torch.empty(cfg.T, cfg.k, dtype=torch.int32, device="cuda")
    w = torch.empty(cfg.T, cfg.k, dtype=torch.float32, device="cuda")
    moe.moe_forward(p, d["x"], d["Wg"], d["bias"], d["W1"], d["W2"], out, ws, idx, w)
    assert moe.moe_get_device_status(ws) == 0
    return out, idx, w, ws


def assert_out_close(got_bf16, ref, what=""):
    got = got_bf16.float().cpu().numpy().astype(np.float64)
    err = np.abs(got - ref)
    bound = ATOL + RTOL * np.abs(ref)
    bad = err > bound
    assert not bad.any(), (f"{what}: {bad.sum()} elements out of tolerance; max |err| "
                           f"{err.max():.3e}")
    return float(err.max())


# ---------------------------------------------------------------------------------------
# router
# ---------------------------------------------------------------------------------------

ROUTE_CASES = [
    # name, T, H, E, k, unscaled gate, zipf bias, gate mode
    ("e8", 300, 256, 8, 2, False, 0.0, 0),
    ("e16_unscaled", 257, 512, 16, 2, True, 0.0, 0),
    ("e64_k8", 130, 384, 64, 8, False, 0.0, 0),
    ("e256_zipf", 70, 448, 256, 8, False, 1.2, 0),
    ("e8_all", 99, 128, 8, 3, False, 0.0, 1),
    ("e40_k40", 33, 64, 40, 40, False, 0.0, 0),
    ("e1024_k33", 9, 64, 1024, 33, False, 0.0, 1),
    # large enough to select each non-narrow tile class of the router
    ("e8_tile", 5000, 192, 8, 2, False, 0.0, 0),
    ("e16_tile", 2500, 320, 16, 2, True, 0.0, 0),
    ("e320_tile", 2100, 128, 320, 8, False, 1.2, 0),
    # selection-only bias (gate 2): SIMT top-k, and the filter's finalize
    ("e8_selbias", 300, 256, 8, 2, False, 1.2, 2),
    ("e64_selbias", 130, 384, 64, 8, False, 1.2, 2),
    ("e256_selbias_tile", 2100, 128, 256, 8, False, 1.2, 2),
    ("e512_max_filter", 600, 192, 512, 16, False, 1.2, 0),
    # small batches with many experts: both decode tile shapes of the sequential router
    ("e256_t64_decode", 64, 512, 256, 8, False, 1.2, 0),
    ("e256_t150_decode", 150, 512, 256, 8, False, 0.0, 0),
    # the one-launch router's thread shapes (2, 4 and 8 threads per token)
    ("e32_k4", 500, 384, 32, 4, False, 1.2, 0),
    ("e24_selbias", 300, 192, 24, 3, False, 1.2, 2),
    ("e32_all", 200, 128, 32, 5, False, 0.0, 1),
    ("e16_t1", 1, 640, 16, 2, False, 0.0, 0),
]


@pytest.fixture(params=[moe.ROUTER_FILTER, moe.ROUTER_SEQUENTIAL], ids=["filter", "sequential"])
def router_mode(request):
    prev = moe.moe_set_router_mode(request.param)
    yield request.param
    moe.moe_set_router_mode(prev)


@pytest.mark.parametrize("case", ROUTE_CASES, ids=[c[0] for c in ROUTE_CASES])
def test_route_bit_exact(case, router_mode):
    name, T, H, E, k, unscaled, zipf, gate = case
    cfg = cfg_small(name, T, H, 64, E, k, gate=gate, gate_std_unscaled=unscaled, zipf_s=zipf)
    inp = synth.make_inputs(cfg, seed=3)
    p = moe.Problem.from_config(cfg)
    ws = alloc_ws(p)
    idx = torch.empty(T, k, dtype=torch.int32, device="cuda")
    w = torch.empty(T, k, dtype=torch.float32, device="cuda")
    bias = inp["bias"].cuda() if inp["bias"] is not None else None
    moe.moe_route(p, inp["x"].cuda(), inp["Wg"].cuda(), bias, idx, w, ws)
    assert moe.moe_get_device_status(ws) == 0
    b = None if bias is None else inp["bias"].numpy()
    # with the selection-only bias the logits exclude it and the top-k adds it to the keys
    logits = oracle.router_logits(bits(inp["x"]), bits(inp["Wg"]),
                                  None if gate == moe.GATE_SELECT_BIAS else b)
    ref_idx, ref_w = oracle.topk_gates(logits, k, gate=gate, bias=b)
    assert np.array_equal(idx.cpu().numpy(), ref_idx)
    np.testing.assert_allclose(w.cpu().numpy(), ref_w, rtol=GATE_RTOL, atol=GATE_ATOL)


def _route(p, x, Wg, bias, T, k):
    ws = alloc_ws(p)
    idx = torch.empty(T, k, dtype=torch.int32, device="cuda")
    w = torch.empty(T, k, dtype=torch.float32, device="cuda")
    moe.moe_route(p, x.cuda(), Wg.cuda(), None if bias is None else bias.cuda(), idx, w, ws)
    assert moe.moe_get_device_status(ws) == 0
    return idx.cpu().numpy(), w.cpu().numpy()


@pytest.mark.parametrize("E,k", [(64, 8), (32, 4), (16, 2), (8, 2)])
@pytest.mark.parametrize("unscaled", [False, True], ids=["scaled", "unscaled"])
def test_route_rounding_level_ties(router_mode, unscaled, E, k):
    """Every expert has the same exact real logit; they differ only in the fp32 rounding of
    the sequential sum (gate columns are one column with pairs of entries swapped where the
    token has equal values), so the choice is made at the last bit of the fp32 logits."""
    T, H = 300, 256
    g = torch.Generator().manual_seed(21)
    x = torch.randn(T, H, generator=g)
    for j in range(6):
        x[:, 2 * j + 1] = x[:, 2 * j]
    x = x.to(torch.bfloat16)
    col = torch.randn(H, generator=g) / (1.0 if unscaled else math.sqrt(H))
    cols = []
    for e in range(E):
        c = col.clone()
        for j in range(6):
            if (e >> j) & 1:
                c[2 * j], c[2 * j + 1] = col[2 * j + 1], col[2 * j]
        cols.append(c)
    Wg = torch.stack(cols, dim=1).to(torch.bfloat16).contiguous()
    p = moe.Problem.make(T, H, 64, E, k)
    got_idx, got_w = _route(p, x, Wg, None, T, k)
    logits = oracle.router_logits(bits(x), bits(Wg), None)
    ref_idx, ref_w = oracle.topk_gates(logits, k)
    assert np.array_equal(got_idx, ref_idx)
    np.testing.assert_allclose(got_w, ref_w, rtol=GATE_RTOL, atol=GATE_ATOL)


@pytest.mark.parametrize("gate", [0, 2], ids=["softmax_topk", "select_bias"])
def test_route_filter_matches_sequential_bitwise(gate):
    """Both router variants give bit-identical indices and gates (the gates are computed from
    the same sequential fp32 logits)."""
    cfg = cfg_small("filter_vs_seq", 1000, 512, 64, 128, 8, zipf_s=1.2, gate=gate)
    inp = synth.make_inputs(cfg, seed=22)
    p = moe.Problem.from_config(cfg)
    res = []
    for mode in (moe.ROUTER_FILTER, moe.ROUTER_SEQUENTIAL):
        prev = moe.moe_set_router_mode(mode)
        try:
            res.append(_route(p, inp["x"], inp["Wg"], inp["bias"], cfg.T, cfg.k))
        finally:
            moe.moe_set_router_mode(prev)
    assert np.array_equal(res[0][0], res[1][0])
    assert np.array_equal(res[0][1].view(np.uint32), res[1][1].view(np.uint32))


@pytest.mark.parametrize("name", ["mixtral", "phi35", "qwen2", "skew", "skew_decode"])
def test_route_filter_matches_sequential_full_size(name):
    """The bench workloads with many experts: filter and sequential routers agree bitwise."""
    cfg = synth.CONFIGS[name]
    inp = synth.make_inputs(cfg, seed=0, device="cuda")
    p = moe.Problem.from_config(cfg)
    res = []
    for mode in (moe.ROUTER_FILTER, moe.ROUTER_SEQUENTIAL):
        prev = moe.moe_set_router_mode(mode)
        try:
            res.append(_route(p, inp["x"], inp["Wg"], inp["bias"], cfg.T, cfg.k))
        finally:
            moe.moe_set_router_mode(prev)
    assert np.array_equal(res[0][0], res[1][0])
    assert np.array_equal(res[0][1].view(np.uint32), res[1][1].view(np.uint32))


def test_route_all_experts_equal(router_mode):
    """Identical gate columns: every logit ties, so the top k are experts 0..k-1 with equal
    gates (every expert is a candidate of the filter)."""
    T, H, E, k = 70, 128, 96, 8
    g = torch.Generator().manual_seed(23)
    x = torch.randn(T, H, generator=g).to(torch.bfloat16)
    col = (torch.randn(H, 1, generator=g) / math.sqrt(H)).to(torch.bfloat16)
    Wg = col.repeat(1, E).contiguous()
    p = moe.Problem.make(T, H, 64, E, k)
    got_idx, got_w = _route(p, x, Wg, None, T, k)
    assert np.array_equal(got_idx, np.tile(np.arange(k, dtype=np.int32), (T, 1)))
    assert np.all(got_w == np.float32(1.0 / k))


def test_route_exact_ties_go_to_lower_id():
    T, H, E, k = 64, 128, 8, 2
    g = torch.Generator().manual_seed(5)
    x = torch.randn(T, H, generator=g).to(torch.bfloat16)
    base = (torch.randn(H, 4, generator=g) / math.sqrt(H)).to(torch.bfloat16)
    Wg = base[:, [0, 1, 2, 3, 3, 2, 1, 0]].contiguous()
    p = moe.Problem.make(T, H, 64, E, k)
    ws = alloc_ws(p)
    idx = torch.empty(T, k, dtype=torch.int32, device="cuda")
    w = torch.empty(T, k, dtype=torch.float32, device="cuda")
    moe.moe_route(p, x.cuda(), Wg.cuda(), None, idx, w, ws)
    got = idx.cpu().numpy()
    mirror = {0: 7, 1: 6, 2: 5, 3: 4}
    for t in range(T):
        assert got[t, 0] < 4 and got[t, 1] == mirror[got[t, 0]]
    assert torch.all(w == 0.5)


# ---------------------------------------------------------------------------------------
# dispatch
# ---------------------------------------------------------------------------------------

def distinct_idx(T, E, k, seed, skew=False):
    rng = np.random.default_rng(seed)
    if skew:
        p = np.arange(1, E + 1, dtype=np.float64) ** -1.2
        p /= p.sum()
        return np.stack([rng.choice(E, size=k, replace=False, p=p) for _ in range(T)]).astype(np.int32)
    return np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)


# T <= 256 takes the one-block dispatch kernel, larger T the three-kernel path
DISPATCH_CASES = [(300, 8, 2, False), (1000, 64, 8, False), (513, 256, 8, True), (1, 4, 1, False),
                  (128, 1, 1, False), (40, 8, 8, False), (2048, 1024, 4, True), (77, 3, 3, False),
                  (256, 1024, 8, True), (256, 8, 2, False), (257, 8, 2, False), (64, 256, 8, True)]


@pytest.mark.parametrize("T,E,k,skew", DISPATCH_CASES)
def test_dispatch_bit_exact(T, E, k, skew):
    H = 64
    p = moe.Problem.make(T, H, 64, E, k)
    ws = alloc_ws(p)
    idx_np = distinct_idx(T, E, k, seed=T * 7 + E, skew=skew)
    ref = oracle.dispatch(idx_np, E)
    pmax = moe.moe_padded_rows_max(p)
    assert pmax == ref["gather_idx"].shape[0] - E * 127 + min(E, T * k) * 127
    dev = dict(counts=torch.full((E,), -7, dtype=torch.int32, device="cuda"),
               offsets=torch.full((E + 1,), -7, dtype=torch.int32, device="cuda"),
               padded_offsets=torch.full((E + 1,), -7, dtype=torch.int32, device="cuda"),
               gather_idx=torch.full((pmax,), -7, dtype=torch.int32, device="cuda"),
               inv_pos=torch.full((T, k), -7, dtype=torch.int32, device="cuda"))
    x = torch.randn(T, H).to(torch.bfloat16)
    x_perm = torch.full((pmax, H), 3.0, dtype=torch.bfloat16, device="cuda")
    moe.moe_dispatch(p, torch.from_numpy(idx_np).cuda(), dev["counts"], dev["offsets"],
                     dev["padded_offsets"], dev["gather_idx"], dev["inv_pos"], ws,
                     x_perm=x_perm, x=x.cuda())
    assert moe.moe_get_device_status(ws) == 0
    for key in ("counts", "offsets", "padded_offsets", "inv_pos"):
        assert np.array_equal(dev[key].cpu().numpy(), ref[key]), key
    gi = dev["gather_idx"].cpu().numpy()
    assert np.array_equal(gi, ref["gather_idx"][:pmax])
    P_pad = int(ref["padded_offsets"][-1])
    xp = x_perm[:P_pad].cpu()
    want = torch.zeros(P_pad, H, dtype=torch.bfloat16)
    valid = torch.from_numpy(gi[:P_pad] >= 0)
    want[valid] = x[torch.from_numpy(gi[:P_pad][gi[:P_pad] >= 0]).long()]
    assert torch.equal(xp, want)


@pytest.mark.parametrize("T", [50, 700])
def test_dispatch_reports_bad_expert_id(T):
    E, k = 8, 2
    p = moe.Problem.make(T, 64, 64, E, k)
    ws = alloc_ws(p)
    idx = torch.from_numpy(distinct_idx(T, E, k, 1)).cuda()
    idx[T - 7, 1] = E + 3
    pmax = moe.moe_padded_rows_max(p)
    bufs = [torch.empty(n, dtype=torch.int32, device="cuda") for n in (E, E + 1, E + 1, pmax)]
    inv = torch.empty(T, k, dtype=torch.int32, device="cuda")
    moe.moe_dispatch(p, idx, *bufs, inv, ws)
    assert moe.moe_get_device_status(ws) == -6
    assert moe.moe_get_device_status(ws) == 0     # read-and-clear


# ---------------------------------------------------------------------------------------
# combine
# ---------------------------------------------------------------------------------------

@pytest.mark.parametrize("T,H,E,k", [(300, 256, 8, 2), (65, 448, 64, 8), (1, 64, 4, 4)])
def test_combine_matches_oracle(T, H, E, k):
    idx = distinct_idx(T, E, k, seed=T + H)
    d = oracle.dispatch(idx, E)
    rows = d["gather_idx"].shape[0]
    ys = (torch.randn(rows, H, generator=torch.Generator().manual_seed(2)) * 0.3).to(torch.bfloat16)
    p = moe.Problem.make(T, H, 64, E, k)
    out = torch.empty(T, H, dtype=torch.bfloat16, device="cuda")
    moe.moe_combine(p, ys.cuda(), torch.from_numpy(d["inv_pos"]).cuda(), out)
    torch.cuda.synchronize()
    ref = oracle.combine(bits(ys), d["inv_pos"])
    got = out.float().cpu().numpy().astype(np.float64)
    assert np.all(np.abs(got - ref) <= 2.0**-8 * np.abs(ref) + 1e-6)


def test_combine_reports_bad_row():
    T, H, k = 10, 64, 2
    p = moe.Problem.make(T, H, 64, 4, k)
    ws = alloc_ws(p)
    ys = torch.ones(20, H, dtype=torch.bfloat16, device="cuda")
    inv = torch.zeros(T, k, dtype=torch.int32, device="cuda")
    inv[3, 1] = 20
    out = torch.empty(T, H, dtype=torch.bfloat16, device="cuda")
    moe.moe_combine(p, ys, inv, out, ws=ws)
    assert moe.moe_get_device_status(ws) == -6
    assert torch.all(out[3] == 1.0) and torch.all(out[0] == 2.0)


# ---------------------------------------------------------------------------------------
# whole layer, small sizes: several tiles, ragged tails, degenerate cases
# ---------------------------------------------------------------------------------------

FWD_CASES = [
    cfg_small("tiny", 256, 256, 512, 8, 2),
    cfg_small("ragged", 300, 192, 320, 8, 2),              # F % 128 == 64, odd T
    cfg_small("many_experts", 200, 256, 256, 64, 8),        # mostly 1-tile experts
    cfg_small("zipf", 160, 320, 192, 32, 4, zipf_s=1.2),    # empty and 0-1 token experts
    cfg_small("one_token", 1, 128, 128, 8, 2),
    cfg_small("k_eq_e", 40, 128, 128, 4, 4),
    cfg_small("single_expert", 130, 128, 256, 1, 1),        # dense FFN
    cfg_small("softmax_all", 100, 128, 128, 8, 2, gate=1),
    cfg_small("gelu", 150, 128, 256, 8, 2, act=1),
    cfg_small("relu", 150, 128, 320, 8, 2, act=2),
    cfg_small("identity", 90, 128, 192, 8, 2, act=3),
    cfg_small("deep_k", 64, 1024, 128, 8, 2),               # long K loop, ring wraps many times
    cfg_small("max_experts", 1500, 128, 64, 1024, 8),       # E at its limit, every expert single-tile
    cfg_small("wide_filter", 700, 192, 128, 512, 6, zipf_s=1.2),  # largest E of the filter router
    # T*k >= 128*E: layer0 reads expert-sorted x rows by TMA with eight epilogue warps (the
    # large-batch path), several m-tiles per expert with a partial last one, ragged N
    cfg_small("sorted_rows", 700, 256, 320, 4, 2),
    cfg_small("sorted_rows_e8", 1100, 192, 384, 8, 2, zipf_s=0.5),
    cfg_small("sorted_rows_gelu", 640, 128, 448, 2, 1, act=1),
]


@pytest.fixture(params=[moe.GEMM_CTA_PAIR, moe.GEMM_SINGLE_CTA, moe.GEMM_FUSED,
                        moe.GEMM_FUSED_LAYERS],
                ids=["cta_pair", "single_cta", "fused", "fused_layers"])
def gemm_mode(request):
    prev = moe.moe_set_gemm_mode(request.param)
    yield request.param
    moe.moe_set_gemm_mode(prev)


@pytest.mark.parametrize("cfg", FWD_CASES, ids=[c.name for c in FWD_CASES])
def test_forward_matches_oracle(cfg, gemm_mode):
    inp = synth.make_inputs(cfg, seed=11)
    out, idx, w, ws = run_forward(cfg, inp)
    b = None if inp["bias"] is None else inp["bias"].numpy()
    ref, ref_idx, ref_w = oracle.moe_forward(bits(inp["x"]), bits(inp["Wg"]), b, bits(inp["W1"]),
                                             bits(inp["W2"]), cfg.k, act=cfg.act, gate=cfg.gate)
    assert np.array_equal(idx.cpu().numpy(), ref_idx)
    np.testing.assert_allclose(w.cpu().numpy(), ref_w, rtol=GATE_RTOL, atol=GATE_ATOL)
    assert_out_close(out, ref, cfg.name)
    out2, _, _, _ = run_forward(cfg, inp, ws)
    assert torch.equal(out, out2), "two identical calls differ"


def test_forward_with_filter_router():
    """The whole layer with the tensor-core filter router forced on a small problem."""
    cfg = cfg_small("filter_fwd", 333, 256, 192, 64, 6, zipf_s=1.2)
    inp = synth.make_inputs(cfg, seed=15)
    prev = moe.moe_set_router_mode(moe.ROUTER_FILTER)
    try:
        out, idx, w, _ = run_forward(cfg, inp)
    finally:
        moe.moe_set_router_mode(prev)
    b = inp["bias"].numpy()
    ref, ref_idx, ref_w = oracle.moe_forward(bits(inp["x"]), bits(inp["Wg"]), b, bits(inp["W1"]),
                                             bits(inp["W2"]), cfg.k)
    assert np.array_equal(idx.cpu().numpy(), ref_idx)
    np.testing.assert_allclose(w.cpu().numpy(), ref_w, rtol=GATE_RTOL, atol=GATE_ATOL)
    assert_out_close(out, ref, cfg.name)


@pytest.mark.parametrize("name", ["skew_small", "skew", "skew_decode"])
def test_work_orders_agree(name):
    """Expert-major and mixed orders only reorder work items: bitwise the same layer output.
    The narrow kernel for single-tile experts computes the same products with the operands
    swapped: within the parity tolerance of the others."""
    cfg = (cfg_small("skew_small", 900, 256, 192, 64, 4, zipf_s=1.2) if name == "skew_small"
           else synth.CONFIGS[name])
    inp = synth.make_inputs(cfg, seed=16, device="cuda")
    outs = {}
    for order in (moe.ORDER_EXPERT, moe.ORDER_MIXED, moe.ORDER_NARROW, moe.ORDER_PHASED):
        prev = moe.moe_set_work_order(order)
        try:
            outs[order] = run_forward(cfg, inp)[0]
        finally:
            moe.moe_set_work_order(prev)
    assert torch.equal(outs[moe.ORDER_EXPERT], outs[moe.ORDER_MIXED])
    a = outs[moe.ORDER_EXPERT].float()
    for order in (moe.ORDER_NARROW, moe.ORDER_PHASED):
        d = (outs[order].float() - a).abs()
        assert bool(torch.all(d <= ATOL + RTOL * a.abs())), (order, float(d.max()))


@pytest.mark.parametrize("order", [0, 1, 2, 3], ids=["expert", "mixed", "narrow", "phased"])
def test_forward_orders_match_oracle(order):
    """A mix of multi-tile and single-tile experts (ragged row counts, some experts empty)
    against the oracle in every work order."""
    cfg = cfg_small("orders", 700, 320, 256, 32, 3, zipf_s=1.5)
    inp = synth.make_inputs(cfg, seed=17)
    prev = moe.moe_set_work_order(order)
    try:
        out, idx, w, _ = run_forward(cfg, inp)
    finally:
        moe.moe_set_work_order(prev)
    b = inp["bias"].numpy()
    ref, ref_idx, _ = oracle.moe_forward(bits(inp["x"]), bits(inp["Wg"]), b, bits(inp["W1"]),
                                         bits(inp["W2"]), cfg.k)
    assert np.array_equal(idx.cpu().numpy(), ref_idx)
    assert_out_close(out, ref, f"order {order}")


def test_forward_with_selection_bias():
    """The whole layer with the selection-only bias (a strong Zipf prior steers the choice,
    the gates ignore it), on the sequential and the filter router."""
    cfg = cfg_small("selbias_fwd", 400, 256, 192, 64, 4, zipf_s=1.5, gate=moe.GATE_SELECT_BIAS)
    inp = synth.make_inputs(cfg, seed=18)
    b = inp["bias"].numpy()
    ref, ref_idx, ref_w = oracle.moe_forward(bits(inp["x"]), bits(inp["Wg"]), b, bits(inp["W1"]),
                                             bits(inp["W2"]), cfg.k, gate=cfg.gate)
    for mode in (moe.ROUTER_SEQUENTIAL, moe.ROUTER_FILTER):
        prev = moe.moe_set_router_mode(mode)
        try:
            out, idx, w, _ = run_forward(cfg, inp)
        finally:
            moe.moe_set_router_mode(prev)
        assert np.array_equal(idx.cpu().numpy(), ref_idx)
        np.testing.assert_allclose(w.cpu().numpy(), ref_w, rtol=GATE_RTOL, atol=GATE_ATOL)
        assert_out_close(out, ref, f"selection bias, router {mode}")


def test_gemm_variants_agree():
    """The single-CTA and CTA-pair grouped GEMMs compute the same layer."""
    cfg = cfg_small("variants", 700, 512, 640, 8, 2)
    inp = synth.make_inputs(cfg, seed=14)
    prev = moe.moe_set_gemm_mode(moe.GEMM_SINGLE_CTA)
    try:
        a, _, _, _ = run_forward(cfg, inp)
        for mode in (moe.GEMM_CTA_PAIR, moe.GEMM_FUSED):
            moe.moe_set_gemm_mode(mode)
            b, _, _, _ = run_forward(cfg, inp)
            d = (a.float() - b.float()).abs()
            assert float(d.max()) <= 2e-2 + 2e-2 * float(a.float().abs().max()), mode
    finally:
        moe.moe_set_gemm_mode(prev)


# The persistent launch that also routes and dispatches (E == 8, T * k >= 128 E, the one-launch
# router): short last h chunk, 8-token groups with idle CTAs, softmax over all experts with
# GELU, the selection-only bias with k = 3, and 128-token groups with two groups on some CTAs.
WHOLE_CASES = [
    cfg_small("wl_e8", 1100, 192, 384, 8, 2, zipf_s=0.5),
    cfg_small("wl_groups8", 1000, 512, 256, 8, 2),
    cfg_small("wl_gelu_all", 1500, 256, 320, 8, 2, act=1, gate=1),
    cfg_small("wl_selbias", 1200, 256, 256, 8, 3, zipf_s=1.5, gate=moe.GATE_SELECT_BIAS),
    cfg_small("wl_two_groups", 20000, 256, 128, 8, 2),
]


@pytest.mark.parametrize("cfg", WHOLE_CASES, ids=[c.name for c in WHOLE_CASES])
def test_whole_layer_launch_matches_oracle_and_separate_launches(cfg):
    """One launch for the whole layer: the routing, gates and output are bitwise those of
    the separate route and dispatch launches, and match the oracle."""
    inp = synth.make_inputs(cfg, seed=19)
    p = moe.Problem.from_config(cfg)
    prev = moe.moe_set_gemm_mode(moe.GEMM_AUTO)
    try:
        assert moe.moe_forward_launches(p) == 1
        one = run_forward(cfg, inp)
        prev_w = moe.moe_set_whole_layer_launch(False)
        try:
            assert moe.moe_forward_launches(p) > 1
            sep = run_forward(cfg, inp)
        finally:
            moe.moe_set_whole_layer_launch(prev_w)
        again = run_forward(cfg, inp, one[3])  # the same workspace again: counters restart
    finally:
        moe.moe_set_gemm_mode(prev)
    for a, b, what in zip(one[:3], sep[:3], ("out", "topk_idx", "topk_w")):
        assert torch.equal(a, b), what
    assert torch.equal(one[0], again[0])
    b = None if inp["bias"] is None else inp["bias"].numpy()
    ref, ref_idx, ref_w = oracle.moe_forward(bits(inp["x"]), bits(inp["Wg"]), b, bits(inp["W1"]),
                                             bits(inp["W2"]), cfg.k, act=cfg.act, gate=cfg.gate)
    assert np.array_equal(one[1].cpu().numpy(), ref_idx)
    np.testing.assert_allclose(one[2].cpu().numpy(), ref_w, rtol=GATE_RTOL, atol=GATE_ATOL)
    assert_out_close(one[0], ref, cfg.name)


def test_forward_all_tokens_on_one_expert():
    cfg = cfg_small("one_hot", 300, 128, 128, 8, 1)
    inp = synth.make_inputs(cfg, seed=12)
    inp["bias"] = torch.tensor([0, 0, 0, 100.0, 0, 0, 0, 0], dtype=torch.float32)
    out, idx, _, _ = run_forward(cfg, inp)
    assert torch.all(idx == 3)
    ref, _, _ = oracle.moe_forward(bits(inp["x"]), bits(inp["Wg"]), inp["bias"].numpy(),
                                   bits(inp["W1"]), bits(inp["W2"]), 1)
    assert_out_close(out, ref, "one_hot")


def test_forward_empty_batch():
    cfg = cfg_small("empty", 0, 128, 128, 8, 2)
    p = moe.Problem.from_config(cfg)
    ws = alloc_ws(p)
    inp = synth.make_inputs(cfg_small("w", 1, 128, 128, 8, 2), seed=1)
    out = torch.empty(0, 128, dtype=torch.bfloat16, device="cuda")
    x = torch.empty(0, 128, dtype=torch.bfloat16, device="cuda")
    moe.moe_forward(p, x, inp["Wg"].cuda(), None, inp["W1"].cuda(), inp["W2"].cuda(), out, ws)
    assert moe.moe_get_device_status(ws) == 0


def test_forward_host_buffers():
    cfg = cfg_small("host", 200, 256, 256, 8, 2)
    inp = synth.make_inputs(cfg, seed=13)
    p = moe.Problem.from_config(cfg)
    ws = alloc_ws(p)
    x_h = inp["x"].pin_memory()
    out_h = torch.empty(cfg.T, cfg.H, dtype=torch.bfloat16).pin_memory()
    moe.moe_forward_host(p, x_h, inp["Wg"].cuda(), None, inp["W1"].cuda(), inp["W2"].cuda(), out_h, ws)
    out_d, _, _, _ = run_forward(cfg, inp)
    assert torch.equal(out_h, out_d.cpu())


def test_forward_host_batches_pipeline():
    """A stream of host batches with overlapped copies gives, batch by batch, exactly the
    outputs of moe_forward on the same inputs (including repeated buffers)."""
    cfg = cfg_small("host_batches", 300, 256, 256, 16, 2)
    base = synth.make_inputs(cfg, seed=19)
    p = moe.Problem.from_config(cfg)
    ws = alloc_ws(p)
    xs = [synth.make_inputs(cfg, seed=19, x_seed=100 + i)["x"].pin_memory() for i in range(5)]
    xs.append(xs[0])                                  # the same input buffer twice
    outs = [torch.empty(cfg.T, cfg.H, dtype=torch.bfloat16).pin_memory() for _ in xs]
    d = {k: (v.cuda() if v is not None else None) for k, v in base.items()}
    moe.moe_forward_host_batches(p, xs, d["Wg"], d["bias"], d["W1"], d["W2"], outs, ws)
    assert moe.moe_get_device_status(ws) == 0
    for i, x in enumerate(xs):
        want = torch.empty(cfg.T, cfg.H, dtype=torch.bfloat16, device="cuda")
        moe.moe_forward(p, x.cuda(), d["Wg"], d["bias"], d["W1"], d["W2"], want, ws)
        assert torch.equal(outs[i], want.cpu()), f"batch {i}"


@pytest.mark.parametrize("with_gate", [True, False], ids=["gated", "ungated"])
def test_forward_shared_matches_oracle(gemm_mode, with_gate):
    """Routed experts plus a shared expert (Fs % 128 == 64, ragged T) against the oracle."""
    cfg = cfg_small("shared", 300, 256, 192, 16, 2, zipf_s=1.2)
    Fs = 320
    inp = synth.make_inputs(cfg, seed=20)
    W1s, W2s, w_sg = synth.make_shared_weights(cfg.H, Fs, 21, gate=with_gate)
    p = moe.Problem.from_config(cfg)
    ws = torch.empty(moe.moe_workspace_size_shared(p, Fs), dtype=torch.uint8, device="cuda")
    d = {k: (v.cuda() if v is not None else None) for k, v in inp.items()}
    out = torch.empty(cfg.T, cfg.H, dtype=torch.bfloat16, device="cuda")
    moe.moe_forward_shared(p, d["x"], d["Wg"], d["bias"], d["W1"], d["W2"], W1s.cuda(), W2s.cuda(),
                           None if w_sg is None else w_sg.cuda(), out, ws)
    assert moe.moe_get_device_status(ws) == 0
    b = inp["bias"].numpy()
    ref, _, _ = oracle.moe_forward(bits(inp["x"]), bits(inp["Wg"]), b, bits(inp["W1"]),
                                   bits(inp["W2"]), cfg.k)
    ref = ref + oracle.shared_tokens(bits(inp["x"]), bits(W1s), bits(W2s),
                                     None if w_sg is None else bits(w_sg), np.arange(cfg.T))
    assert_out_close(out, ref, f"shared, gate {with_gate}")


def test_forward_shared_full_size_qwen2():
    """The Qwen2-shaped layer with a 20480-wide shared expert (Qwen2-57B-A14B's), on a token
    sample checked one by one against the oracle."""
    cfg = synth.CONFIGS["qwen2"]
    Fs = 20480
    inp = synth.make_inputs(cfg, seed=0, device="cuda")
    W1s, W2s, w_sg = synth.make_shared_weights(cfg.H, Fs, 22, device="cuda")
    p = moe.Problem.from_config(cfg)
    ws = torch.empty(moe.moe_workspace_size_shared(p, Fs), dtype=torch.uint8, device="cuda")
    out = torch.empty(cfg.T, cfg.H, dtype=torch.bfloat16, device="cuda")
    moe.moe_forward_shared(p, inp["x"], inp["Wg"], inp["bias"], inp["W1"], inp["W2"], W1s, W2s,
                           w_sg, out, ws)
    assert moe.moe_get_device_status(ws) == 0
    host = {k: (bits(v) if v is not None and v.dtype == torch.bfloat16 else v) for k, v in inp.items()}
    toks = np.unique(np.random.default_rng(3).choice(cfg.T, size=12, replace=False)).astype(np.int32)
    toks = np.concatenate([toks, np.array([cfg.T - 1], np.int32)])
    b = None if inp["bias"] is None else inp["bias"].cpu().numpy()
    ref, _, _ = oracle.moe_tokens(host["x"], host["Wg"], b, host["W1"], host["W2"], cfg.k, toks,
                                  act=cfg.act, gate=cfg.gate)
    ref = ref + oracle.shared_tokens(host["x"], bits(W1s), bits(W2s), bits(w_sg), toks)
    assert_out_close(out[torch.from_numpy(toks).long().cuda()], ref, "qwen2 + shared")


# ---------------------------------------------------------------------------------------
# full-size workloads (the bench configurations), launched exactly as the bench does
# ---------------------------------------------------------------------------------------

FULL = ["mixtral", "phi35", "qwen2", "skew", "skew_decode"]
N_RANDOM_TOKENS = 2048
_FULL_REF = {}  # workload -> oracle routing and the reference rows of its token sample


def full_size_sample(ref_idx, T, E, seed=0):
    """Tokens whose layer output is checked against the oracle at full size:
      - every token of the four least-loaded active experts (their tiles, including their
        last, partial m-tile, are checked row by row);
      - for every active expert, the token of the first row of each of its 128-row m-tiles
        and of its last row, so that every m-tile of every expert (every tile position of
        the expert-major GEMM order, and each expert's partial last tile) is covered;
      - a seeded random subset of min(T, 2048) tokens.
    The layer is computed token by token (Comet §2.1 "MoE Structure"), so a subset check is
    a check of those tokens' rows in full."""
    counts = np.bincount(ref_idx.reshape(-1), minlength=E)
    active = np.nonzero(counts)[0]
    rare = active[np.argsort(counts[active], kind="stable")][:4]
    toks = [np.nonzero((ref_idx == e).any(axis=1))[0] for e in rare]
    for e in active:
        rows = np.nonzero((ref_idx == e).any(axis=1))[0]   # ascending token id = row order
        toks.append(rows[::128])
        toks.append(rows[-1:])
    rng = np.random.default_rng(seed)
    toks.append(rng.choice(T, size=min(T, N_RANDOM_TOKENS), replace=False))
    return np.unique(np.concatenate(toks).astype(np.int32))


def full_size_reference(name, cfg, inp):
    """Oracle routing of the whole batch and oracle output rows of the token sample,
    computed once per workload and shared by the GEMM modes."""
    if name not in _FULL_REF:
        host = {k: (bits(v) if v is not None and v.dtype == torch.bfloat16 else v)
                for k, v in inp.items()}
        b = None if inp["bias"] is None else inp["bias"].cpu().numpy()
        logits = oracle.router_logits(host["x"], host["Wg"], b)
        ref_idx, ref_w = oracle.topk_gates(logits, cfg.k, gate=cfg.gate)
        toks = full_size_sample(ref_idx, cfg.T, cfg.E)
        ref, _, _ = oracle.moe_tokens(host["x"], host["Wg"], b, host["W1"], host["W2"], cfg.k, toks,
                                      act=cfg.act, gate=cfg.gate)
        _FULL_REF[name] = (ref_idx, ref_w, toks, ref)
    return _FULL_REF[name]


@pytest.mark.parametrize("name", FULL)
def test_full_size_config(name, gemm_mode):
    cfg = synth.CONFIGS[name]
    inp = synth.make_inputs(cfg, seed=0, device="cuda")
    out, idx, w, ws = run_forward(cfg, inp)
    ref_idx, ref_w, toks, ref = full_size_reference(name, cfg, inp)
    # routing in full, bit-exact
    assert np.array_equal(idx.cpu().numpy(), ref_idx)
    np.testing.assert_allclose(w.cpu().numpy(), ref_w, rtol=GATE_RTOL, atol=GATE_ATOL)
    # output rows of the token sample
    assert_out_close(out[torch.from_numpy(toks).long().cuda()], ref, f"{name}: {len(toks)} tokens")
