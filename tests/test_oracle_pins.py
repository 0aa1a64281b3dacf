"""Pins of the CPU oracle against facts fixed outside the oracle itself.

Every pin is one of: a hand-worked closed form (tests/golden), exact integer arithmetic,
a floating-point error bound, a mathematical identity, a special case that reduces to a
dense matmul (numpy), or brute force over all experts. Each is chosen so that a plausible
slip in the oracle (a dropped term, a transposed operand, a wrong index, a wrong tie-break,
gate and up columns swapped) fails at least one of them.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from mixture_experts_layer_forward_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
ACTS = {"swiglu": oracle.ACT_SWIGLU, "gelu_tanh": oracle.ACT_GELU_TANH, "relu": oracle.ACT_RELU,
        "identity": oracle.ACT_IDENTITY}
GATES = {"softmax_topk": oracle.GATE_SOFTMAX_TOPK, "softmax_all": oracle.GATE_SOFTMAX_ALL}


def bf16(a):
    """Exact small values -> bf16 bit patterns (asserts exact representability)."""
    t = torch.tensor(np.asarray(a, dtype=np.float64), dtype=torch.float64)
    b = t.to(torch.bfloat16)
    assert torch.equal(b.to(torch.float64), t), "value not exact in bf16"
    return synth.bf16_bits(b)


def widen(u16):
    return synth.from_bf16_bits(u16).to(torch.float64).numpy()


def rand_bf16(shape, seed, std=1.0):
    g = torch.Generator().manual_seed(seed)
    return synth.bf16_bits((torch.randn(shape, generator=g) * std).to(torch.bfloat16))


def distinct_topk_idx(T, E, k, seed):
    rng = np.random.default_rng(seed)
    return np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)


# ------------------------------------------------------------------------------------
# hand-worked closed forms
# ------------------------------------------------------------------------------------

def test_golden_hand_worked_cases(oracle_lib):
    with open(os.path.join(GOLDEN, "hand_worked.json")) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        x, Wg, W1, W2 = (bf16(c[n]) for n in ("x", "Wg", "W1", "W2"))
        out, idx, w = oracle.moe_forward(x, Wg, None, W1, W2, c["k"], act=ACTS[c["act"]],
                                         gate=GATES[c["gate"]], lib=oracle_lib)
        assert idx.tolist() == c["expected_idx"], c["name"]
        np.testing.assert_allclose(w, c["expected_w"], rtol=1e-14, atol=0, err_msg=c["name"])
        np.testing.assert_allclose(out, c["expected_out"], rtol=1e-14, atol=1e-15, err_msg=c["name"])
        # the per-token definition path agrees as well
        out2, idx2, w2 = oracle.moe_tokens(x, Wg, None, W1, W2, c["k"], np.arange(c["T"]),
                                           act=ACTS[c["act"]], gate=GATES[c["gate"]], lib=oracle_lib)
        assert idx2.tolist() == c["expected_idx"]
        np.testing.assert_allclose(out2, c["expected_out"], rtol=1e-14, atol=1e-15)


def test_round_to_bf16_hand_cases(oracle_lib):
    cases = {
        1.0: 1.0,
        1 + 2**-8: 1.0,                      # tie, even neighbour is 1.0
        1 + 3 * 2**-8: 1 + 2**-6,            # tie, even neighbour is 1 + 2/128
        1 + 2**-8 + 2**-20: 1 + 2**-7,       # just above the tie
        -3.0: -3.0,
        0.1: 0.10009765625,                  # bf16 0x3DCD
        -(2**-100) * 1.00390625: -(2**-100), # tie at a small exponent
    }
    for v, want in cases.items():
        assert oracle.round_to_bf16(v, lib=oracle_lib) == want, v
    # fp32 inputs: torch's float32 -> bfloat16 conversion (one nearest-even rounding) agrees,
    # on random values and on the fp32 neighbours of bf16 midpoints
    rng = np.random.default_rng(4)
    r = np.ldexp(rng.uniform(1, 2, 3000), rng.integers(-60, 60, 3000)) * rng.choice([-1, 1], 3000)
    mids = np.ldexp(2.0 * np.arange(128, 256) + 1, -8).astype(np.float32)  # (2m+1)/256 in [1, 2)
    v32 = np.concatenate([r.astype(np.float32), mids, np.nextafter(mids, np.float32(2)),
                          np.nextafter(mids, np.float32(0))])
    lib_vals = torch.from_numpy(v32).to(torch.bfloat16).to(torch.float64).numpy()
    got = np.array([oracle.round_to_bf16(float(v), lib=oracle_lib) for v in v32])
    np.testing.assert_array_equal(got, lib_vals)


# ------------------------------------------------------------------------------------
# router logits: exact integers, summation order, error bound
# ------------------------------------------------------------------------------------

def test_router_logits_small_integers_exact(oracle_lib):
    rng = np.random.default_rng(1)
    T, H, E = 7, 96, 5
    xi = rng.integers(-4, 5, size=(T, H))
    wi = rng.integers(-4, 5, size=(H, E))
    bi = rng.integers(-8, 9, size=E).astype(np.float32)
    got = oracle.router_logits(bf16(xi), bf16(wi), bi, lib=oracle_lib)
    want = (xi @ wi).astype(np.float64) + bi      # exact integers, well below 2^24
    np.testing.assert_array_equal(got.astype(np.float64), want)


def test_router_logits_sequential_fp32_order(oracle_lib):
    # x . w with w = 1 and x = [2^24, 1, 1, -2^24]: a single fp32 accumulator walking h
    # upward loses both ones (2^24 + 1 rounds back to 2^24) and ends at 0; the exact sum
    # is 2, and the order [1, 1, 2^24, -2^24] keeps them (result 2).
    x = bf16([[2**24, 1, 1, -(2**24)], [1, 1, 2**24, -(2**24)]])
    w = bf16(np.ones((4, 1)))
    got = oracle.router_logits(x, w, None, lib=oracle_lib)
    assert got[0, 0] == 0.0 and got[1, 0] == 2.0


def test_router_logits_within_fp32_error_bound(oracle_lib):
    T, H, E = 32, 1024, 16
    x = rand_bf16((T, H), 11)
    Wg = rand_bf16((H, E), 12, std=1 / math.sqrt(H))
    bias = np.linspace(-1, 1, E).astype(np.float32)
    got = oracle.router_logits(x, Wg, bias, lib=oracle_lib).astype(np.float64)
    xf, wf = widen(x), widen(Wg)
    exact = xf @ wf + bias.astype(np.float64)
    absdot = np.abs(xf) @ np.abs(wf)
    u = 2.0**-24
    gamma = (H + 1) * u / (1 - (H + 1) * u)       # H products summed, plus the bias add
    bound = gamma * (absdot + np.abs(bias)) + 1e-30
    assert np.all(np.abs(got - exact) <= bound)
    # and it really is fp32 (not a wider accumulator): some entries differ from exact
    assert np.any(got != exact)


# ------------------------------------------------------------------------------------
# top-k selection and gates
# ------------------------------------------------------------------------------------

def test_topk_order_and_ties(oracle_lib):
    l = np.array([[1.0, 3.0, 3.0, 2.0, -0.0, 0.0]], np.float32)
    idx, _ = oracle.topk_gates(l, 6, lib=oracle_lib)
    assert idx.tolist() == [[1, 2, 3, 0, 4, 5]]       # equal values: lower id first; -0 == +0
    idx, _ = oracle.topk_gates(l, 2, lib=oracle_lib)
    assert idx.tolist() == [[1, 2]]


def test_router_ties_from_duplicated_gate_columns(oracle_lib):
    T, H = 64, 128
    x = rand_bf16((T, H), 3)
    base = rand_bf16((H, 4), 4, std=1 / math.sqrt(H))
    Wg = np.ascontiguousarray(base[:, [0, 1, 2, 3, 3, 2, 1, 0]])   # experts 4..7 copy 3..0
    logits = oracle.router_logits(x, Wg, None, lib=oracle_lib)
    assert np.array_equal(logits[:, :4], logits[:, [7, 6, 5, 4]])
    idx, w = oracle.topk_gates(logits, 2, lib=oracle_lib)
    # the best logit always appears twice, so both selected experts share one value and
    # the pair is (lower copy, higher copy)
    mirror = {0: 7, 1: 6, 2: 5, 3: 4}
    for t in range(T):
        a, b = idx[t]
        assert a < 4 and b == mirror[a]
        assert w[t, 0] == w[t, 1] == 0.5


def test_gates_match_full_softmax_then_renormalise(oracle_lib):
    T, E, k = 50, 12, 3
    rng = np.random.default_rng(5)
    logits = (rng.standard_normal((T, E)) * 3).astype(np.float32)
    idx, w = oracle.topk_gates(logits, k, lib=oracle_lib)
    l64 = logits.astype(np.float64)
    full = np.exp(l64 - l64.max(axis=1, keepdims=True))
    full /= full.sum(axis=1, keepdims=True)
    sel = np.take_along_axis(full, idx.astype(np.int64), axis=1)
    np.testing.assert_allclose(w, sel / sel.sum(axis=1, keepdims=True), rtol=1e-13)
    np.testing.assert_allclose(w.sum(axis=1), 1.0, rtol=0, atol=k * 2**-52)
    assert np.all(np.diff(w, axis=1) <= 0)
    # indices are the k largest, in descending order
    ref = np.argsort(-l64, axis=1, kind="stable")[:, :k]
    assert np.array_equal(idx, ref)
    # SOFTMAX_ALL keeps the full-softmax values
    idx2, w2 = oracle.topk_gates(logits, k, gate=oracle.GATE_SOFTMAX_ALL, lib=oracle_lib)
    assert np.array_equal(idx2, idx)
    np.testing.assert_allclose(w2, sel, rtol=1e-13)
    # k = 1 gives a weight of exactly one
    _, w1 = oracle.topk_gates(logits, 1, lib=oracle_lib)
    assert np.all(w1 == 1.0)


def test_selection_bias_closed_form(oracle_lib):
    """SELECT_BIAS: the bias decides which experts are selected, the gates come from the
    logits without it (hand-worked: raw logits [3, 1, 2, 0], bias [0, 5, 0, 4] give keys
    [3, 6, 2, 4], so experts 1 then 3; gates softmax([1, 0]) shifted by its max, 1)."""
    x = bf16([[1.0, 1.0]])
    Wg = bf16([[2.0, 0.0, 1.0, 0.0], [1.0, 1.0, 1.0, 0.0]])      # logits [3, 1, 2, 0]
    bias = np.array([0.0, 5.0, 0.0, 4.0], np.float32)
    raw = oracle.router_logits(x, Wg, None, lib=oracle_lib)
    assert raw.tolist() == [[3.0, 1.0, 2.0, 0.0]]
    idx, w = oracle.topk_gates(raw, 2, gate=oracle.GATE_SELECT_BIAS, bias=bias, lib=oracle_lib)
    assert idx.tolist() == [[1, 3]]
    e1 = math.exp(-1.0)
    np.testing.assert_allclose(w, [[1 / (1 + e1), e1 / (1 + e1)]], rtol=1e-15)
    # SOFTMAX_TOPK on the biased logits selects the same experts but gates by [6, 4]
    idx0, w0 = oracle.topk_gates(oracle.router_logits(x, Wg, bias, lib=oracle_lib), 2,
                                 lib=oracle_lib)
    e2 = math.exp(-2.0)
    assert idx0.tolist() == [[1, 3]]
    np.testing.assert_allclose(w0, [[1 / (1 + e2), e2 / (1 + e2)]], rtol=1e-15)
    # ties of the keys still go to the lower id; no bias gives SOFTMAX_TOPK exactly
    tie = np.array([[1.0, 0.0, 2.0]], np.float32)
    idx_t, _ = oracle.topk_gates(tie, 1, gate=oracle.GATE_SELECT_BIAS,
                                 bias=np.array([1.0, 2.0, 0.0], np.float32), lib=oracle_lib)
    assert idx_t.tolist() == [[0]]                               # keys [2, 2, 2]
    rng = np.random.default_rng(9)
    l = rng.standard_normal((20, 7)).astype(np.float32)
    a = oracle.topk_gates(l, 3, gate=oracle.GATE_SELECT_BIAS, lib=oracle_lib)
    b = oracle.topk_gates(l, 3, lib=oracle_lib)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


# ------------------------------------------------------------------------------------
# dispatch: counting sort against a library stable sort, plus invariants
# ------------------------------------------------------------------------------------

@pytest.mark.parametrize("T,E,k,m_tile", [(300, 8, 2, 128), (97, 64, 8, 128), (5, 16, 3, 4),
                                          (1000, 3, 3, 128), (0, 4, 1, 128)])
def test_dispatch_matches_stable_sort(oracle_lib, T, E, k, m_tile):
    idx = distinct_topk_idx(T, E, k, seed=T + E) if T else np.zeros((0, k), np.int32)
    d = oracle.dispatch(idx, E, m_tile=m_tile, lib=oracle_lib)
    flat = idx.reshape(-1)
    counts = np.bincount(flat, minlength=E)
    assert np.array_equal(d["counts"], counts)
    assert d["counts"].sum() == T * k
    assert np.array_equal(d["offsets"], np.concatenate([[0], np.cumsum(counts)]))
    padded = -(-counts // m_tile) * m_tile
    poff = np.concatenate([[0], np.cumsum(padded)])
    assert np.array_equal(d["padded_offsets"], poff)
    order = np.argsort(flat, kind="stable")            # pair ids sorted by expert, token-stable
    gi = d["gather_idx"]
    for e in range(E):
        pairs = order[d["offsets"][e]:d["offsets"][e + 1]]
        rows = gi[poff[e]:poff[e] + counts[e]]
        assert np.array_equal(rows, pairs // k)
        assert np.all(np.diff(rows) > 0)                  # ascending token id
        assert np.all(gi[poff[e] + counts[e]:poff[e + 1]] == -1)
    assert np.all(gi[poff[E]:] == -1)
    inv = d["inv_pos"]
    for t in range(T):
        for j in range(k):
            r = inv[t, j]
            assert gi[r] == t and poff[flat[t * k + j]] <= r < poff[flat[t * k + j] + 1]
    # tiles: one per m_tile block of each expert's rows
    nt = int(np.sum(-(-counts // m_tile)))
    assert d["num_tiles"] == nt
    want = [(e, poff[e] + i * m_tile, min(m_tile, counts[e] - i * m_tile))
            for e in range(E) for i in range(-(-counts[e] // m_tile))]
    got = list(zip(d["tile_expert"], d["tile_row0"], d["tile_nvalid"]))
    assert [tuple(map(int, g)) for g in got] == [tuple(map(int, w_)) for w_ in want]


def test_permute_then_unpermute_is_identity(oracle_lib):
    T, H, E, k = 200, 24, 10, 4
    x = rand_bf16((T, H), 9)
    idx = distinct_topk_idx(T, E, k, seed=9)
    d = oracle.dispatch(idx, E, lib=oracle_lib)
    gi = d["gather_idx"]
    xp = np.zeros((gi.shape[0], H), np.uint16)
    xp[gi >= 0] = x[gi[gi >= 0]]
    for j in range(k):
        assert np.array_equal(xp[d["inv_pos"][:, j]], x)


# ------------------------------------------------------------------------------------
# experts and whole layer
# ------------------------------------------------------------------------------------

def _np_act(act, z):
    """The activations from torch's library implementations (fp64), not retyped here."""
    zt = torch.from_numpy(np.ascontiguousarray(z, dtype=np.float64))
    if act == oracle.ACT_GELU_TANH:
        return torch.nn.functional.gelu(zt, approximate="tanh").numpy()
    if act == oracle.ACT_RELU:
        return torch.relu(zt).numpy()
    return z


def _np_ffn(x64, W1e, W2e, act, F):
    z = x64 @ W1e
    if act == oracle.ACT_SWIGLU:
        g = torch.from_numpy(np.ascontiguousarray(z[:, :F]))
        a = torch.nn.functional.silu(g).numpy() * z[:, F:]
    else:
        a = _np_act(act, z)
    return a @ W2e


@pytest.mark.parametrize("act", [oracle.ACT_SWIGLU, oracle.ACT_GELU_TANH, oracle.ACT_RELU,
                                 oracle.ACT_IDENTITY])
def test_single_expert_top1_is_dense_ffn(oracle_lib, act):
    T, H, F = 9, 64, 40
    c = 2 * F if act == oracle.ACT_SWIGLU else F
    x = rand_bf16((T, H), 21)
    Wg = rand_bf16((H, 1), 22)
    W1 = rand_bf16((1, H, c), 23, std=1 / math.sqrt(H))
    W2 = rand_bf16((1, F, H), 24, std=1 / math.sqrt(F))
    out, idx, w = oracle.moe_forward(x, Wg, None, W1, W2, 1, act=act, lib=oracle_lib)
    assert np.all(idx == 0) and np.all(w == 1.0)
    want = _np_ffn(widen(x), widen(W1[0]), widen(W2[0]), act, F)
    np.testing.assert_allclose(out, want, rtol=1e-12, atol=1e-12)


def test_identity_experts_reproduce_x(oracle_lib):
    T, H, E, k = 40, 16, 5, 3
    x = rand_bf16((T, H), 31)
    Wg = rand_bf16((H, E), 32, std=1 / math.sqrt(H))
    eye = np.broadcast_to(np.eye(H), (E, H, H))
    W = bf16(eye)
    out, _, w = oracle.moe_forward(x, Wg, None, W, W, k, act=oracle.ACT_IDENTITY, lib=oracle_lib)
    np.testing.assert_allclose(out, widen(x), rtol=4e-16 * k, atol=0)


@pytest.mark.parametrize("act,gate,use_bias", [(oracle.ACT_SWIGLU, oracle.GATE_SOFTMAX_TOPK, False),
                                               (oracle.ACT_SWIGLU, oracle.GATE_SOFTMAX_ALL, True),
                                               (oracle.ACT_GELU_TANH, oracle.GATE_SOFTMAX_TOPK, True),
                                               (oracle.ACT_RELU, oracle.GATE_SOFTMAX_TOPK, False),
                                               (oracle.ACT_SWIGLU, oracle.GATE_SELECT_BIAS, True)])
def test_layer_equals_dense_masked_sum_over_all_experts(oracle_lib, act, gate, use_bias):
    """Brute force: run every expert on every token (numpy matmuls), then mask with the
    gate matrix; routing from fp64 logits with a full stable sort."""
    T, H, F, E, k = 48, 64, 32, 6, 2
    c = 2 * F if act == oracle.ACT_SWIGLU else F
    x = rand_bf16((T, H), 41)
    Wg = rand_bf16((H, E), 42)            # unscaled: well separated logits
    W1 = rand_bf16((E, H, c), 43, std=1 / math.sqrt(H))
    W2 = rand_bf16((E, F, H), 44, std=1 / math.sqrt(F))
    bias = np.linspace(0.5, -0.5, E).astype(np.float32) if use_bias else None
    out, idx, w = oracle.moe_forward(x, Wg, bias, W1, W2, k, act=act, gate=gate, lib=oracle_lib)

    xf = widen(x)
    # the fp32 logits are pinned by the router tests above; from here on everything is
    # recomputed independently: full stable sort, full softmax, every expert on every token
    sel_bias = gate == oracle.GATE_SELECT_BIAS
    l32 = oracle.router_logits(x, Wg, None if sel_bias else bias, lib=oracle_lib)
    l = l32.astype(np.float64)
    l_exact = xf @ widen(Wg) + (0 if (bias is None or sel_bias) else bias.astype(np.float64))
    np.testing.assert_allclose(l, l_exact, rtol=0, atol=1e-3)
    # selection keys: the logits, or with a selection bias their fp32 sum with it
    keys = (l32 + bias).astype(np.float64) if sel_bias else l
    sel = np.argsort(-keys, axis=1, kind="stable")[:, :k]
    G = np.zeros((T, E))
    p = np.exp(l - l.max(axis=1, keepdims=True))
    for t in range(T):
        if gate == oracle.GATE_SOFTMAX_ALL:
            G[t, sel[t]] = p[t, sel[t]] / p[t].sum()
        else:
            G[t, sel[t]] = p[t, sel[t]] / p[t, sel[t]].sum()
    dense = np.stack([_np_ffn(xf, widen(W1[e]), widen(W2[e]), act, F) for e in range(E)], axis=1)
    want = np.einsum("te,teh->th", G, dense)
    assert np.array_equal(idx, sel)
    np.testing.assert_allclose(out, want, rtol=1e-10, atol=1e-12)
    toks = np.array([0, 5, 17, 47], np.int32)
    out_t, idx_t, _ = oracle.moe_tokens(x, Wg, bias, W1, W2, k, toks, act=act, gate=gate, lib=oracle_lib)
    assert np.array_equal(idx_t, sel[toks])
    np.testing.assert_allclose(out_t, want[toks], rtol=1e-10, atol=1e-12)


def test_combine_is_row_gather_sum(oracle_lib):
    T, H, E, k = 77, 40, 9, 3
    idx = distinct_topk_idx(T, E, k, seed=51)
    d = oracle.dispatch(idx, E, lib=oracle_lib)
    ys = rand_bf16((d["gather_idx"].shape[0], H), 52)
    got = oracle.combine(ys, d["inv_pos"], lib=oracle_lib)
    want = widen(ys)[d["inv_pos"]].sum(axis=1)
    np.testing.assert_allclose(got, want, rtol=1e-15, atol=0)


def test_round_a_bf16_flag_changes_only_by_rounding(oracle_lib):
    T, H, F, E, k = 16, 64, 64, 4, 2
    x = rand_bf16((T, H), 61)
    Wg = rand_bf16((H, E), 62)
    W1 = rand_bf16((E, H, 2 * F), 63, std=1 / math.sqrt(H))
    W2 = rand_bf16((E, F, H), 64, std=1 / math.sqrt(F))
    a, _, _ = oracle.moe_forward(x, Wg, None, W1, W2, k, lib=oracle_lib)
    b, _, _ = oracle.moe_forward(x, Wg, None, W1, W2, k, round_a_bf16=True, lib=oracle_lib)
    assert not np.array_equal(a, b)
    np.testing.assert_allclose(a, b, rtol=0, atol=2**-8 * np.abs(a).max() * 2)


# ------------------------------------------------------------------------------------
# shared expert (a model feature outside the pages)
# ------------------------------------------------------------------------------------

def test_shared_expert_term(oracle_lib):
    """g_t * FFN_s(x_t): without a gate vector it is the dense SwiGLU FFN (numpy), with a zero
    gate vector exactly half of it, and the gate is the logistic function of x . w_sg
    (hand-checked on exact small integers)."""
    T, H, Fs = 11, 64, 48
    x = rand_bf16((T, H), 61)
    W1s = rand_bf16((H, 2 * Fs), 62, std=1 / math.sqrt(H))
    W2s = rand_bf16((Fs, H), 63, std=1 / math.sqrt(Fs))
    toks = np.arange(T, dtype=np.int32)
    dense = _np_ffn(widen(x), widen(W1s), widen(W2s), oracle.ACT_SWIGLU, Fs)
    full = oracle.shared_tokens(x, W1s, W2s, None, toks, lib=oracle_lib)
    np.testing.assert_allclose(full, dense, rtol=1e-10, atol=1e-12)
    half = oracle.shared_tokens(x, W1s, W2s, bf16(np.zeros(H)), toks, lib=oracle_lib)
    np.testing.assert_array_equal(half, 0.5 * full)
    # gate on exact integers: x_0 . w_sg = 1*2 + 1*(-3) = -1 for the first token below
    xi = np.zeros((2, H)); xi[0, :2] = [1, 1]; xi[1, :3] = [2, 0, 1]
    wsg = np.zeros(H); wsg[:3] = [2, -3, 1]                      # z = [-1, 5]
    xb = bf16(xi)
    g_ffn = oracle.shared_tokens(xb, W1s, W2s, None, np.array([0, 1], np.int32), lib=oracle_lib)
    got = oracle.shared_tokens(xb, W1s, W2s, bf16(wsg), np.array([0, 1], np.int32), lib=oracle_lib)
    for i, z in enumerate([-1.0, 5.0]):
        np.testing.assert_allclose(got[i], g_ffn[i] / (1 + math.exp(-z)), rtol=1e-14, atol=1e-300)


# ---------------------------------------------------------------------------------------
# FP8 (e4m3) experts (a precision variant outside the pages)
# ---------------------------------------------------------------------------------------

def _e4m3_table():
    """Every e4m3 code's value written out from the format's definition (sign, 4-bit
    exponent with bias 7, 3-bit mantissa, subnormals at exponent 0, S.1111.111 NaN), built
    here with Python integer arithmetic, independently of the oracle's decoder."""
    vals = []
    for c in range(256):
        s, ef, m = c >> 7, (c >> 3) & 15, c & 7
        if ef == 15 and m == 7:
            vals.append(math.nan)
            continue
        v = m * 2.0 ** -9 if ef == 0 else (8 + m) * 2.0 ** (ef - 10)
        vals.append(-v if s else v)
    return np.array(vals)


def test_e4m3_decode_known_codes(oracle_lib):
    table = _e4m3_table()
    got = oracle.e4m3_decode(np.arange(256, dtype=np.uint8), lib=oracle_lib)
    np.testing.assert_array_equal(np.isnan(got), np.isnan(table))
    ok = ~np.isnan(table)
    np.testing.assert_array_equal(got[ok], table[ok])
    # a few values stated outright
    assert got[0x38] == 1.0 and got[0x7E] == 448.0 and got[0x01] == 2.0 ** -9
    assert got[0x08] == 2.0 ** -6 and got[0x40] == 2.0 and got[0x3F] == 1.875
    assert np.isnan(got[0x7F]) and np.isnan(got[0xFF]) and got[0xB8] == -1.0
    # the positive finite codes are strictly increasing
    assert np.all(np.diff(got[:0x7F]) > 0)
    # and torch's float8_e4m3fn type reads every finite code the same way
    lib_vals = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64)
    np.testing.assert_array_equal(got[ok], lib_vals.numpy()[ok])


def test_e4m3_encode_is_nearest_ties_to_even(oracle_lib):
    """Brute force over every finite code: the nearest value, ties to the even code,
    magnitudes above 448 saturate, on the codes' values, their midpoints, the floats just
    either side of each midpoint, random values and the special values."""
    table = _e4m3_table()
    pos = table[:0x7F]  # codes 0x00..0x7E, increasing
    mids = (pos[:-1] + pos[1:]) / 2
    mids32 = mids.astype(np.float32)
    assert np.all(mids32.astype(np.float64) == mids)  # the midpoints are exact in fp32
    rng = np.random.default_rng(7)
    v = np.concatenate([
        pos, mids32, np.nextafter(mids32, np.float32(np.inf)), np.nextafter(mids32, np.float32(0)),
        rng.uniform(-500, 500, 20000), rng.uniform(-0.02, 0.02, 20000),
        np.ldexp(rng.uniform(1, 2, 5000), rng.integers(-12, 10, 5000)),
        [448.0, 449.0, 463.9, 464.0, 480.0, 1e6, 2.0 ** -10, 3 * 2.0 ** -11]]).astype(np.float32)
    v = np.concatenate([v, -v])
    got = oracle.e4m3_encode(v, lib=oracle_lib)
    a = np.abs(v.astype(np.float64))
    d = np.abs(a[:, None] - pos[None, :])
    best = d.min(axis=1, keepdims=True)
    cand = d == best
    # among equally near codes take the even one (at most two are equally near)
    code = np.where(cand & (np.arange(0x7F)[None, :] % 2 == 0), np.arange(0x7F)[None, :], 999).min(axis=1)
    code = np.where(cand.sum(axis=1) == 1, d.argmin(axis=1), code)
    code = np.where(a > 448.0, 0x7E, code)
    want = (code | np.where(np.signbit(v), 0x80, 0)).astype(np.uint8)
    np.testing.assert_array_equal(got, want)
    # torch's float32 -> float8_e4m3fn conversion (nearest, ties to even) agrees in range
    inr = np.abs(v) <= 448.0
    lib_codes = torch.from_numpy(v[inr]).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(got[inr], lib_codes)
    specials = np.array([np.inf, -np.inf, np.nan, -0.0, 0.0], np.float32)
    sg = oracle.e4m3_encode(specials, lib=oracle_lib)
    assert list(sg[:2]) == [0x7E, 0xFE] and (sg[2] & 0x7F) == 0x7F and list(sg[3:]) == [0x80, 0x00]


def test_fp8_row_quantisation_worked_example(oracle_lib):
    """Row [100, 1, -2, 0]: r = 448/100 = 4.48 -> 448 (0x7E), 4.48 -> 4.5 (0x49),
    -8.96 -> -9 (0xD1), 0 (0x00); scale 100/448 in fp32. A zero row keeps scale 1."""
    q, s = oracle.quant_rows_fp8(bf16([[100, 1, -2, 0], [0, 0, 0, 0]]), lib=oracle_lib)
    assert list(q[0]) == [0x7E, 0x49, 0xD1, 0x00] and list(q[1]) == [0, 0, 0, 0]
    assert s[0] == np.float32(100) / np.float32(448) and s[1] == 1.0


def test_fp8_column_quantisation_worked_example(oracle_lib):
    """W [1, K=3, N=2], columns (100, 1, -2) and (0.5, -0.25, 0.125): per-column scales and
    the transposed (K contiguous) code layout. Column 1: r = 896 -> 448 (0x7E),
    -224 (0xF6), 112 (0x6E)."""
    W = bf16([[[100, 0.5], [1, -0.25], [-2, 0.125]]])
    q, s = oracle.quant_cols_fp8(W, lib=oracle_lib)
    assert q.shape == (1, 2, 3)
    assert list(q[0, 0]) == [0x7E, 0x49, 0xD1] and list(q[0, 1]) == [0x7E, 0xF6, 0x6E]
    assert s[0, 0] == np.float32(100) / np.float32(448) and s[0, 1] == np.float32(0.5) / np.float32(448)


def _fp8_layer(seed, T, H, F, E, k, act):
    g = torch.Generator().manual_seed(seed)
    w1c = 2 * F if act == oracle.ACT_SWIGLU else F
    x = rand_bf16((T, H), seed)
    Wg = rand_bf16((H, E), seed + 1, 1 / math.sqrt(H))
    # columns of very different size (factors 1/8 .. 2), so a scale taken from the wrong
    # column or row is far off
    c1 = 2.0 ** (np.arange(w1c) % 5 - 3)
    c2 = 2.0 ** (np.arange(H) % 5 - 3)
    W1 = (torch.randn(E, H, w1c, generator=g) / math.sqrt(H) * torch.from_numpy(c1).float())
    W2 = (torch.randn(E, F, H, generator=g) / math.sqrt(F) * torch.from_numpy(c2).float())
    return x, Wg, synth.bf16_bits(W1.to(torch.bfloat16)), synth.bf16_bits(W2.to(torch.bfloat16))


def test_fp8_h_is_held_in_bf16_before_its_row_quantisation(oracle_lib):
    """Hand-worked: one token x = (1, 1, 1), one expert, identity activation, H = 3, F = 2.
    x codes 448 each, s_x = fl32(1/448). W1 column 0 = (448, 0, 0): codes (448, 0, 0),
    s = 1, so z0 = 448^2 * s_x = 448 (1 + 4.5e-8). W1 column 1 = (1, 1/16, 146 * 2^-22):
    r = 448, codes (448, 28, 2^-6) (146 * 2^-22 * 448 = 0.01559 rounds to the smallest
    normal), s = fl32(1/448), so z1 = 476.015625 / 448 (1 + 9e-8) = 1.0625349.
    h in bf16: (448, 1.0625), so amax = 448, r_h = s_h = 1 and 1.0625 is a tie between the
    e4m3 values 1 and 1.125 that goes to the even code, 1. W2 column 0 = (0, 1) picks h1:
    out[0] = 1 * 448 * fl32(1/448) = 1 (1 + 4.5e-8). Held in fp32 instead, amax would be
    fl32(z0) > 448, r_h < 1 and h1 * r_h = 1.0625349 would take the code 1.125. W2 column 1 =
    (1, 0) picks h0: out[1] = 448 (1 + 4.5e-8); column 2 is zero (scale 1, codes 0)."""
    x = bf16([[1, 1, 1]])
    Wg = bf16([[1], [0], [0]])
    W1 = bf16([[[448, 1], [0, 1 / 16], [0, 146 * 2.0 ** -22]]])      # [E, H, F]
    W2 = bf16([[[0, 1, 0], [1, 0, 0]]])                              # [E, F, H]
    W1q, s1 = oracle.quant_cols_fp8(W1, lib=oracle_lib)
    W2q, s2 = oracle.quant_cols_fp8(W2, lib=oracle_lib)
    assert list(W1q[0, 1]) == [0x7E, 0x5E, 0x08]                     # 448, 28, 2^-6
    out, idx, w = oracle.moe_tokens_fp8(x, Wg, None, W1q, s1, W2q, s2, 1, np.arange(1),
                                        act=oracle.ACT_IDENTITY, lib=oracle_lib)
    assert idx[0, 0] == 0 and w[0, 0] == 1.0
    assert abs(out[0, 0] - 1.0) < 1e-6, out[0, 0]                    # not 1.125
    assert abs(out[0, 1] - 448.0) < 1e-3 and out[0, 2] == 0.0


@pytest.mark.parametrize("act", [oracle.ACT_SWIGLU, oracle.ACT_RELU])
def test_fp8_layer_is_close_to_bf16_layer(oracle_lib, act):
    """The e4m3 layer equals the bf16 layer up to the quantisation error: each code is within
    2^-4 relative of its value (3 mantissa bits), so the outputs agree to a few percent."""
    T, H, F, E, k = 24, 128, 96, 4, 2
    x, Wg, W1, W2 = _fp8_layer(3, T, H, F, E, k, act)
    W1q, s1 = oracle.quant_cols_fp8(W1, lib=oracle_lib)
    W2q, s2 = oracle.quant_cols_fp8(W2, lib=oracle_lib)
    toks = np.arange(T)
    ref, ridx, _ = oracle.moe_tokens(x, Wg, None, W1, W2, k, toks, act=act, lib=oracle_lib)
    got, gidx, _ = oracle.moe_tokens_fp8(x, Wg, None, W1q, s1, W2q, s2, k, toks, act=act,
                                        lib=oracle_lib)
    np.testing.assert_array_equal(gidx, ridx)
    rel = np.linalg.norm(got - ref) / np.linalg.norm(ref)
    assert rel < 0.08, rel


@pytest.mark.parametrize("act", [oracle.ACT_IDENTITY, oracle.ACT_RELU])
def test_fp8_layer_scales_exactly_with_the_input(oracle_lib, act):
    """One expert (gate 1): with a positively homogeneous activation, x -> 2^j x leaves every
    code unchanged and multiplies every scale, hence the output, by exactly 2^j."""
    T, H, F, E, k = 8, 64, 64, 1, 1
    x, Wg, W1, W2 = _fp8_layer(5, T, H, F, E, k, act)
    W1q, s1 = oracle.quant_cols_fp8(W1, lib=oracle_lib)
    W2q, s2 = oracle.quant_cols_fp8(W2, lib=oracle_lib)
    toks = np.arange(T)
    out, _, _ = oracle.moe_tokens_fp8(x, Wg, None, W1q, s1, W2q, s2, k, toks, act=act, lib=oracle_lib)
    x8 = bf16(widen(x) * 8.0)
    out8, _, _ = oracle.moe_tokens_fp8(x8, Wg, None, W1q, s1, W2q, s2, k, toks, act=act, lib=oracle_lib)
    np.testing.assert_array_equal(out8, 8.0 * out)
    assert np.abs(out).max() > 0


# ---------------------------------------------------------------------------------------
# Backward pass (training; beyond the pages)
# ---------------------------------------------------------------------------------------

def _autograd_grads(x, Wg, bias, W1, W2, dy, k, act, gate, idx):
    """Gradients of sum(dy * out) by torch autograd (float64) of the layer written with the
    selection fixed to idx: a derivative the oracle's hand-written backward does not share."""
    t = lambda a: torch.from_numpy(widen(a)).requires_grad_(True)
    X, G, A, B = t(x), t(Wg), t(W1), t(W2)
    b = torch.from_numpy(np.asarray(bias, np.float64)).requires_grad_(True) if bias is not None else None
    logits = X @ G
    if b is not None and gate != oracle.GATE_SELECT_BIAS:
        logits = logits + b
    sel = torch.from_numpy(idx.astype(np.int64))
    w = torch.softmax(torch.gather(logits, 1, sel), dim=1)
    F = W2.shape[1]
    out = torch.zeros_like(X)
    for j in range(k):
        for e in range(W1.shape[0]):
            rows = (sel[:, j] == e).nonzero().flatten()
            if rows.numel() == 0:
                continue
            z = X[rows] @ A[e]
            if act == oracle.ACT_SWIGLU:
                a = torch.nn.functional.silu(z[:, :F]) * z[:, F:]
            elif act == oracle.ACT_RELU:
                a = torch.relu(z)
            elif act == oracle.ACT_GELU_TANH:
                a = torch.nn.functional.gelu(z, approximate="tanh")
            else:
                a = z
            out = out.index_add(0, rows, w[rows, j:j + 1] * (a @ B[e]))
    loss = (out * torch.from_numpy(widen(dy))).sum()
    params = [X, G, A, B] + ([b] if b is not None else [])
    grads = torch.autograd.grad(loss, params, allow_unused=True)
    names = ["dx", "dWg", "dW1", "dW2"] + (["dbias"] if b is not None else [])
    return {n: (g.numpy() if g is not None else np.zeros(p.shape)) for n, g, p in zip(names, grads, params)}


@pytest.mark.parametrize("act,gate,use_bias", [
    (oracle.ACT_SWIGLU, oracle.GATE_SOFTMAX_TOPK, True),
    (oracle.ACT_SWIGLU, oracle.GATE_SELECT_BIAS, True),
    (oracle.ACT_GELU_TANH, oracle.GATE_SOFTMAX_TOPK, False),
    (oracle.ACT_RELU, oracle.GATE_SOFTMAX_TOPK, True),
], ids=["swiglu_bias", "swiglu_select_bias", "gelu", "relu_bias"])
def test_backward_matches_autograd(oracle_lib, act, gate, use_bias):
    T, H, F, E, k = 20, 32, 24, 6, 2
    w1c = 2 * F if act == oracle.ACT_SWIGLU else F
    x = rand_bf16((T, H), 31)
    Wg = rand_bf16((H, E), 32, 0.5)
    W1 = rand_bf16((E, H, w1c), 33, 1 / math.sqrt(H))
    W2 = rand_bf16((E, F, H), 34, 1 / math.sqrt(F))
    dy = rand_bf16((T, H), 35)
    bias = np.random.default_rng(36).normal(0, 0.5, E).astype(np.float32) if use_bias else None
    g = oracle.moe_backward(x, Wg, bias, W1, W2, dy, k, act=act, gate=gate, lib=oracle_lib)
    logits = oracle.router_logits(x, Wg, None if gate == oracle.GATE_SELECT_BIAS else bias,
                                  lib=oracle_lib)
    idx, _ = oracle.topk_gates(logits, k, gate=gate, bias=bias, lib=oracle_lib)
    ref = _autograd_grads(x, Wg, bias, W1, W2, dy, k, act, gate, idx)
    # the oracle's gates come from fp32 logits, autograd's from fp64 ones: ~1e-7 relative
    for name in ref:
        np.testing.assert_allclose(g[name], ref[name], rtol=1e-5, atol=1e-6, err_msg=name)
    if use_bias and gate == oracle.GATE_SELECT_BIAS:
        assert np.all(g["dbias"] == 0)
    assert np.abs(g["dW1"]).max() > 0 and np.abs(g["dWg"]).max() > 0


def test_backward_dx_tokens_equals_full_backward(oracle_lib):
    T, H, F, E, k = 16, 32, 16, 4, 2
    x = rand_bf16((T, H), 41)
    Wg = rand_bf16((H, E), 42)
    W1 = rand_bf16((E, H, 2 * F), 43, 1 / math.sqrt(H))
    W2 = rand_bf16((E, F, H), 44, 1 / math.sqrt(F))
    dy = rand_bf16((T, H), 45)
    full = oracle.moe_backward(x, Wg, None, W1, W2, dy, k, lib=oracle_lib)
    toks = np.array([3, 0, 15, 7])
    part = oracle.moe_backward_dx_tokens(x, Wg, None, W1, W2, dy, k, toks, lib=oracle_lib)
    np.testing.assert_array_equal(part, full["dx"][toks])
