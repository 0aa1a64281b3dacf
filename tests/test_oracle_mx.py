"""Pins of the oracle's block-scaled FP8 (MX) form, on CPU: e4m3 codes with one e8m0
power-of-two scale per 32 values along K, the smallest 2^X with amax / 2^X <= 448 (so no
element saturates), elements e4m3(v / 2^X). The expected values below are worked by hand
from that rule; the properties (scaling by powers of two, the e4m3 error bound, identity
experts) hold for any correct implementation of it. No GPU; no CUDA path for this form
exists yet."""
import functools
import math

import numpy as np
import pytest

import oracle
from mixture_experts_layer_forward_b200 import synth


class _Bound:
    """The oracle's functions bound to one build of its library (the session's, or a
    deliberately broken copy that tests/test_oracle_mutants.py plants a slip in)."""

    def __init__(self, lib):
        self._lib = lib

    def __getattr__(self, name):
        f = getattr(oracle, name)
        return functools.partial(f, lib=self._lib) if callable(f) else f


def deq(q, s, O):
    """Values of MX codes q [rows, K] with scale bytes s [rows, K / 32]."""
    v = O.e4m3_decode(q)
    scale = np.array([[O.e8m0_decode(b) for b in row] for row in s])
    return v * np.repeat(scale, 32, axis=1)


def test_e8m0_decode(oracle_lib):
    O = _Bound(oracle_lib)
    assert O.e8m0_decode(127) == 1.0
    assert O.e8m0_decode(0) == 2.0 ** -127
    assert O.e8m0_decode(254) == 2.0 ** 127
    assert O.e8m0_decode(120) == 2.0 ** -7
    assert math.isnan(O.e8m0_decode(255))


def test_hand_worked_blocks(oracle_lib):
    O = _Bound(oracle_lib)
    # 32 x 3.0: floor(log2 3) = 1, X = -7 (byte 120); 3 * 2^7 = 384 = 1.5 * 2^8: exponent
    # field 15, mantissa 4 -> code 0x7C; decodes back to 3.0 exactly
    q, s = O.mx_quant_rows_f32(np.full((1, 32), 3.0, np.float32))
    assert s[0, 0] == 120 and np.all(q == 0x7C)
    assert np.all(deq(q, s, O) == 3.0)
    # no saturation: amax 1.9375, and 1.9375 * 2^8 = 496 > 448, so X = -7 (byte 120), not -8;
    # 1.9375 * 128 = 248 = 128 * 1.9375: mantissa 7.5 ties to the even 8, which carries to
    # 256 -> 0x78 (decodes to 2.0); 1.0 -> 128 -> 0x70; 0.5 -> 64 -> 0x68; 0 -> 0x00
    v = np.zeros((1, 32), np.float32)
    v[0, :4] = [1.9375, 1.0, 0.5, 0.0]
    q, s = O.mx_quant_rows_f32(v)
    assert s[0, 0] == 120
    assert list(q[0, :4]) == [0x78, 0x70, 0x68, 0x00]
    assert deq(q, s, O)[0, 0] == 2.0
    # amax exactly 448 * 2^-8 = 1.75: X = -8 keeps it (byte 119), code 0x7E
    v[0, 0] = 1.75
    q, s = O.mx_quant_rows_f32(v)
    assert s[0, 0] == 119 and q[0, 0] == 0x7E
    # a block of zeros takes the smallest scale (byte 0), codes 0
    q, s = O.mx_quant_rows_f32(np.zeros((1, 32), np.float32))
    assert s[0, 0] == 0 and np.all(q == 0)
    # amax 8.0 -> X = -5 (byte 122); -5.25 * 32 = -168 = -128 * 1.3125: mantissa 2.5 ties to
    # the even 2 -> -160 -> code 0x80 | (14 << 3) | 2 = 0xF2, decoding to -5.0
    v = np.zeros((1, 32), np.float32)
    v[0, 0], v[0, 1] = 8.0, -5.25
    q, s = O.mx_quant_rows_f32(v)
    assert s[0, 0] == 122 and q[0, 0] == 0x78 and q[0, 1] == 0xF2
    assert deq(q, s, O)[0, 1] == -5.0
    # a subnormal element: amax 1 (X = -8), 2^-15 * 256 = 2^-7 = 4 * 2^-9 -> code 4, exact
    v = np.zeros((1, 32), np.float32)
    v[0, 0], v[0, 5] = 1.0, 2.0 ** -15
    q, s = O.mx_quant_rows_f32(v)
    assert q[0, 5] == 4 and deq(q, s, O)[0, 5] == 2.0 ** -15
    # each block has its own scale: a second block with amax 64 (X = -2, byte 125)
    v = np.ones((1, 64), np.float32)
    v[0, 32:] = 64.0
    q, s = O.mx_quant_rows_f32(v)
    assert list(s[0]) == [119, 125]


def test_power_of_two_scaling_moves_only_the_scale(oracle_lib):
    O = _Bound(oracle_lib)
    rng = np.random.default_rng(5)
    v = rng.standard_normal((8, 64)).astype(np.float32)
    q0, s0 = O.mx_quant_rows_f32(v)
    for j in (-12, -1, 1, 9):
        q, s = O.mx_quant_rows_f32(v * np.float32(2.0 ** j))
        assert np.array_equal(q, q0)
        assert np.array_equal(s.astype(int), s0.astype(int) + j)


def test_element_error_bound(oracle_lib):
    """Each element within half an e4m3 step of its scaled value: relative 2^-4 in the normal
    range, 2^-10 absolute (times the scale) below it; every block's amax lands in (224, 448]
    times its scale, so nothing saturates and the top binade is used."""
    O = _Bound(oracle_lib)
    rng = np.random.default_rng(6)
    v = (rng.standard_normal((64, 128)) * np.exp(rng.uniform(-6, 6, (64, 1)))).astype(np.float32)
    q, s = O.mx_quant_rows_f32(v)
    d = deq(q, s, O)
    scale = np.repeat(np.array([[O.e8m0_decode(b) for b in row] for row in s]), 32, axis=1)
    a = np.abs(v.astype(np.float64)) / scale
    err = np.abs(d - v.astype(np.float64)) / scale
    normal = a >= 2.0 ** -6
    assert np.all(err[normal] <= a[normal] * 2.0 ** -4)
    assert np.all(err[~normal] <= 2.0 ** -10)
    amax = a.reshape(64, 4, 32).max(axis=2)
    assert np.all(amax <= 448.0) and np.all(amax > 224.0)


def _bits(t):
    return synth.bf16_bits(t)


def test_identity_experts_reproduce_the_block_round_trip(oracle_lib):
    """E = 1, k = 1, identity activation, W1 = W2 = I: the layer returns dequant(MX(x))
    exactly (each output column sees one weight block holding 1.0; h is bf16-exact and its
    re-quantisation repeats x's codes and scales). A wrong block index, a scale taken from
    another block or a transposed operand breaks this."""
    O = _Bound(oracle_lib)
    import torch

    T, H = 16, 64
    rng = np.random.default_rng(7)
    x = torch.from_numpy((rng.standard_normal((T, H)) * 3).astype(np.float32)).to(torch.bfloat16)
    Wg = torch.ones(H, 1, dtype=torch.bfloat16)
    eye = torch.eye(H, dtype=torch.bfloat16).reshape(1, H, H)
    W1q, W1s = O.mx_quant_cols(_bits(eye))
    W2q, W2s = O.mx_quant_cols(_bits(eye))
    out, idx, w = O.moe_tokens_mx(_bits(x), _bits(Wg), None, W1q, W1s, W2q, W2s, 1,
                                       np.arange(T), act=O.ACT_IDENTITY)
    assert np.all(idx == 0) and np.all(w == 1.0)
    q, s = O.mx_quant_rows(_bits(x))
    assert np.array_equal(out, deq(q, s, O))
    # the block structure matters: a per-row scale (the row-scaled FP8 form) differs
    qr, sr = O.quant_rows_fp8(_bits(x))
    assert not np.array_equal(out, O.e4m3_decode(qr) * sr[:, None].astype(np.float64))


def test_h_is_rounded_to_bf16_before_its_block_quantisation(oracle_lib):
    """The activation h is stored in bf16 and quantised from there. Hand-worked: x = (1, 2^-4,
    2^-9, 0, ...) is exact in MX (block scale 2^-8: codes for 256, 16 and 0.5); W1's column 0
    sums x's first three entries, so z_0 = 1 + 2^-4 + 2^-9, and with the identity
    activation h_0 = z_0. bf16 keeps 1.0625 (2^-9 is below half its step of 2^-7); h's block
    scale is 2^-8 and 1.0625 * 256 = 272 lies halfway between e4m3's 256 and 288, so ties
    to even give 256 and W2 = I returns 1.0. Quantising the unrounded 272.5 would give 288,
    i.e. 1.125."""
    O = _Bound(oracle_lib)
    import torch

    H = F = 32
    x = torch.zeros(2, H, dtype=torch.bfloat16)
    x[0, :3] = torch.tensor([1.0, 2.0 ** -4, 2.0 ** -9])
    Wg = torch.ones(H, 1, dtype=torch.bfloat16)
    W1 = torch.zeros(1, H, F, dtype=torch.bfloat16)
    W1[0, :3, 0] = 1.0
    W2 = torch.eye(F, dtype=torch.bfloat16).reshape(1, F, H)
    W1q, W1s = O.mx_quant_cols(_bits(W1))
    W2q, W2s = O.mx_quant_cols(_bits(W2))
    out, _, _ = O.moe_tokens_mx(_bits(x), _bits(Wg), None, W1q, W1s, W2q, W2s, 1, np.arange(2),
                                act=O.ACT_IDENTITY)
    assert out[0, 0] == 1.0
    assert np.all(out[0, 1:] == 0.0) and np.all(out[1] == 0.0)


@pytest.mark.parametrize("act", [oracle.ACT_IDENTITY, oracle.ACT_RELU])
def test_layer_scales_exactly_with_the_input(oracle_lib, act):
    """W_g = 0: every logit is 0, so each token takes experts 0 and 1 (ties to the lower id)
    with gates 1/2 whatever x is. With a positively homogeneous activation, x -> 2^3 x leaves
    every code of x and of h unchanged and raises every scale byte by 3, so the output is
    exactly 8 times the original (the bf16 rounding of h commutes with a power of two)."""
    O = _Bound(oracle_lib)
    cfg = synth.LayerConfig("mx_h", T=16, H=64, F=96, E=4, k=2, act=act)
    inp = synth.make_inputs(cfg, seed=9)
    Wg = np.zeros((cfg.H, cfg.E), np.uint16)
    W1q, W1s = O.mx_quant_cols(_bits(inp["W1"]))
    W2q, W2s = O.mx_quant_cols(_bits(inp["W2"]))
    toks = np.arange(cfg.T)
    out, idx, w = O.moe_tokens_mx(_bits(inp["x"]), Wg, None, W1q, W1s, W2q, W2s, cfg.k, toks,
                                  act=act)
    assert np.all(idx == [0, 1]) and np.all(w == 0.5)
    x8 = _bits((inp["x"].float() * 8.0).to(inp["x"].dtype))
    out8, _, _ = O.moe_tokens_mx(x8, Wg, None, W1q, W1s, W2q, W2s, cfg.k, toks, act=act)
    np.testing.assert_array_equal(out8, 8.0 * out)
    assert np.abs(out).max() > 0


def test_layer_close_to_the_exact_layer(oracle_lib):
    """The MX layer against the exact (bf16 operands, fp64) layer on random data. Four
    operands are rounded to e4m3 (x, W1, h, W2), each with a relative error of at most 2^-4
    and an rms of at most 2^-4 / sqrt(3) = 0.036; independent, they add to about
    sqrt(4) * 0.036 = 0.072 of the output's rms. Measured on seeds 8-11: 0.065-0.068 rms and
    0.31-0.49 of the rms at the worst element. A scale taken from the wrong block, a dropped
    scale or a transposed block index is off by powers of two and fails both bounds."""
    O = _Bound(oracle_lib)
    cfg = synth.LayerConfig("mx", T=64, H=128, F=96, E=4, k=2)
    inp = synth.make_inputs(cfg, seed=8)
    W1q, W1s = O.mx_quant_cols(_bits(inp["W1"]))
    W2q, W2s = O.mx_quant_cols(_bits(inp["W2"]))
    toks = np.arange(cfg.T)
    out, idx, _ = O.moe_tokens_mx(_bits(inp["x"]), _bits(inp["Wg"]), None, W1q, W1s, W2q,
                                       W2s, cfg.k, toks)
    ref, ref_idx, _ = O.moe_forward(_bits(inp["x"]), _bits(inp["Wg"]), None, _bits(inp["W1"]),
                                         _bits(inp["W2"]), cfg.k)
    assert np.array_equal(idx, ref_idx)       # the routing is the bf16 path's
    rms = np.sqrt(np.mean(ref ** 2))
    assert np.max(np.abs(out - ref)) <= 0.6 * rms
    assert np.sqrt(np.mean((out - ref) ** 2)) <= 0.085 * rms


def test_k_must_be_a_multiple_of_32(oracle_lib):
    O = _Bound(oracle_lib)
    with pytest.raises(ValueError):
        O.mx_quant_rows_f32(np.zeros((1, 48), np.float32))
