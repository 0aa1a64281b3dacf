"""The oracle's pins must catch plausible mistakes in the oracle itself.

Each mutant below plants one slip in a copy of oracle/moe_oracle.c (a dropped term, a
transposed operand, a wrong index, order or tie-break, a wrong constant or sign, a wider
accumulator), builds it, and runs tests/test_oracle_pins.py and tests/test_oracle_mx.py
against that build. Every mutant must make at least one pin fail. Mutations that leave the result mathematically unchanged
(for example dropping the max shift of the softmax) are not mistakes and are not listed.
"""
import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor
from pathlib import Path

import pytest

import oracle

ROOT = Path(__file__).resolve().parents[1]
SRC = ROOT / "oracle" / "moe_oracle.c"

PIN_FILES = ("test_oracle_pins.py", "test_oracle_mx.py")

MUTANTS = [
    ("router_wider_accumulator", "float acc = 0.0f;", "double acc = 0.0;"),
    ("router_h_descending",
     "for (int h = 0; h < H; ++h) {\n                float p",
     "for (int h = H - 1; h >= 0; --h) {\n                float p"),
    ("router_drops_bias", "if (bias) acc = acc + bias[e];", ""),
    ("router_transposed_gate", "bf16_to_float(Wg[(size_t)h * E + e])",
     "bf16_to_float(Wg[(size_t)e * H + h])"),
    ("topk_ties_to_higher_id", "sel_key(gate, l, bias, e) > sel_key(gate, l, bias, best)",
     "sel_key(gate, l, bias, e) >= sel_key(gate, l, bias, best)"),
    ("gates_over_all_experts", "if (gate == ORACLE_GATE_SOFTMAX_ALL) {",
     "if (gate != ORACLE_GATE_SOFTMAX_ALL) {"),
    ("silu_wrong_sign", "z / (1.0 + exp(-z))", "z / (1.0 + exp(z))"),
    ("swiglu_gate_up_swapped", "silu(z[f]) * z[F + f]", "silu(z[F + f]) * z[f]"),
    ("gelu_wrong_constant", "0.044715", "0.04715"),
    ("w2_transposed", "y[n] += a * (double)bf16_to_float(wrow[n]);",
     "y[n] += a * (double)bf16_to_float(W2e[(size_t)n * F + f]);"),
    ("ffn_first_x_only", "double xh = (double)bf16_to_float(xrow[h]);",
     "double xh = (double)bf16_to_float(xrow[0]);"),
    ("combine_drops_gate", "s += w[(size_t)t * k + j] * y[(size_t)r * H + n];",
     "s += y[(size_t)r * H + n];"),
    ("token_path_drops_gate", "o[n] += w[j] * y[n];", "o[n] += y[n];"),
    ("dispatch_pads_down", "((counts[e] + m_tile - 1) / m_tile) * m_tile",
     "(counts[e] / m_tile) * m_tile"),
    ("dispatch_not_stable",
     "for (int t = 0; t < T; ++t) {\n        for (int j = 0; j < k; ++j) {\n            int e = idx[(size_t)t * k + j];\n            int r = poff[e] + cursor[e];",
     "for (int t = T - 1; t >= 0; --t) {\n        for (int j = 0; j < k; ++j) {\n            int e = idx[(size_t)t * k + j];\n            int r = poff[e] + cursor[e];"),
    ("bf16_ties_away_from_zero", "nearbyint(scaled)", "round(scaled)"),
    ("bf16_seven_bits", "ldexp(m, 8)", "ldexp(m, 7)"),
    ("select_bias_logits_keep_bias",
     "oracle_router_logits(T, H, E, x, Wg, gate == ORACLE_GATE_SELECT_BIAS ? NULL : bias, logits);",
     "oracle_router_logits(T, H, E, x, Wg, bias, logits);"),
    ("select_bias_ignored_in_selection", "? l[e] + bias[e] : l[e];", "? l[e] : l[e];"),
    ("shared_gate_wrong_sign", "g = 1.0 / (1.0 + exp(-z));", "g = 1.0 / (1.0 + exp(z));"),
    ("e4m3_ties_away_from_zero", "code = ((ex + 7) << 3) + m;",
     "code = ((ex + 7) << 3) + (int)round((ldexp(a, -ex) - 1.0) * 8.0);"),
    ("e4m3_no_subnormals", "code = (int)nearbyint(ldexp(a, 9));", "code = 0;"),
    ("e4m3_exponent_bias_8", "const int ex = e - 1;", "const int ex = e - 2;"),
    ("fp8_scale_for_e5m2_range", "*r = 448.0f / amax;", "*r = 240.0f / amax;"),
    ("fp8_weight_scale_per_row", "for (int kk = 0; kk < K; ++kk) v[kk] = bf16_to_float(col[(size_t)kk * N]);",
     "for (int kk = 0; kk < K; ++kk) v[kk] = bf16_to_float(col[(size_t)kk]);"),
    ("fp8_h_scale_dropped", "y[n] = acc * (double)sh * (double)s2[n];", "y[n] = acc * (double)s2[n];"),
    ("fp8_x_scale_dropped", "z[c] = acc * (double)sx * (double)s1[c];", "z[c] = acc * (double)s1[c];"),
    ("fp8_w1_scale_of_column_0", "z[c] = acc * (double)sx * (double)s1[c];", "z[c] = acc * (double)sx * (double)s1[0];"),
    ("fp8_gate_up_swapped",
     "silu(z[f]) * z[f + F] : act_apply(act, z[f]);\n        hf[f] = (float)oracle_round_to_bf16(a);\n    }\n    const float sh",
     "silu(z[f + F]) * z[f] : act_apply(act, z[f]);\n        hf[f] = (float)oracle_round_to_bf16(a);\n    }\n    const float sh"),
    ("fp8_token_path_drops_gate", "y, z, hf, hq);\n                for (int n = 0; n < H; ++n) o[n] += y[n] * w[j];",
     "y, z, hf, hq);\n                for (int n = 0; n < H; ++n) o[n] += y[n];"),
    ("mx_token_path_drops_gate", "y, z, hf, hq, hs);\n                for (int n = 0; n < H; ++n) o[n] += y[n] * w[j];",
     "y, z, hf, hq, hs);\n                for (int n = 0; n < H; ++n) o[n] += y[n];"),
    ("fp8_h_not_rounded_to_bf16", "hf[f] = (float)oracle_round_to_bf16(a);\n    }\n    const float sh",
     "hf[f] = (float)a;\n    }\n    const float sh"),
    ("bwd_silu_derivative_drops_term", "const double dg = da[f] * u * s * (1.0 + g * (1.0 - s));",
     "const double dg = da[f] * u * s;"),
    ("bwd_up_gradient_uses_up", "const double du = da[f] * g * s;", "const double du = da[f] * u * s;"),
    ("bwd_softmax_not_centred", "const double dl = (dw[j] - wdw) * w[j];", "const double dl = dw[j] * w[j];"),
    ("bwd_dbias_with_selection_bias", "if (gate != ORACLE_GATE_SELECT_BIAS) dbias[e] += dl;",
     "dbias[e] += dl;"),
    ("bwd_dW2_without_gate", "drow[n] += a[f] * gscale * (double)bf16_to_float(dyr[n]);",
     "drow[n] += a[f] * (double)bf16_to_float(dyr[n]);"),
    ("bwd_dx_tokens_not_centred", "const double dl = w[j] * (dw[j] - wdw);", "const double dl = w[j] * dw[j];"),
    ("mx_scale_saturating_rule", "if (ldexp(amax, -X) > 448.0) X += 1;", ""),
    ("mx_scale_exponent_of_e5m2", "X = (e - 1) - 8;", "X = (e - 1) - 15;"),
    ("mx_e8m0_bias_128", "return ldexp(1.0, (int)b - 127);", "return ldexp(1.0, (int)b - 128);"),
    ("mx_dot_scale_of_block_0",
     "acc += part * oracle_e8m0_decode(sa[b]) * oracle_e8m0_decode(sb[b]);",
     "acc += part * oracle_e8m0_decode(sa[0]) * oracle_e8m0_decode(sb[b]);"),
    ("mx_dot_weight_scale_dropped",
     "acc += part * oracle_e8m0_decode(sa[b]) * oracle_e8m0_decode(sb[b]);",
     "acc += part * oracle_e8m0_decode(sa[b]);"),
    ("mx_weight_blocks_along_n", "v[i] = bf16_to_float(col[(size_t)(b * 32 + i) * N]);",
     "v[i] = bf16_to_float(col[(size_t)(b * 32 + i)]);"),
    ("mx_w1_scales_of_expert_0", "W1s + (size_t)e * w1_cols * (H / 32), W2q",
     "W1s, W2q"),
    ("mx_w2_scale_stride_of_codes", "W2s + (size_t)e * H * (F / 32), y, z",
     "W2s + (size_t)e * H * F / 64, y, z"),
    ("mx_gate_up_swapped",
     "silu(z[f]) * z[f + F] : act_apply(act, z[f]);\n        hf[f] = (float)oracle_round_to_bf16(a);\n    }\n    for (int b",
     "silu(z[f + F]) * z[f] : act_apply(act, z[f]);\n        hf[f] = (float)oracle_round_to_bf16(a);\n    }\n    for (int b"),
    ("mx_h_not_rounded_to_bf16",
     "        hf[f] = (float)oracle_round_to_bf16(a);\n    }\n    for (int b = 0; b < F / 32; ++b)",
     "        hf[f] = (float)a;\n    }\n    for (int b = 0; b < F / 32; ++b)"),
    ("shared_ffn_uses_gate_half_only", "ffn_row(H, Fs, ORACLE_ACT_SWIGLU, 0, xr, W1s, W2s, y, scratch);",
     "ffn_row(H, Fs, ORACLE_ACT_GELU_TANH, 0, xr, W1s, W2s, y, scratch);"),
]


def _run_mutant(tmp_path, name, old, new):
    text = SRC.read_text()
    if text.count(old) != 1:
        return f"{name}: the mutation site is missing or not unique"
    d = tmp_path / name
    d.mkdir()
    src = d / "moe_oracle.c"
    src.write_text(text.replace(old, new))
    lib = oracle.build(force=True, src=src, out=d / "liboracle_mutant.so")
    env = dict(os.environ, ORACLE_LIB_UNDER_TEST=str(lib), OMP_NUM_THREADS="2")
    r = subprocess.run([sys.executable, "-m", "pytest", *[str(ROOT / "tests" / f) for f in PIN_FILES],
                        "-x", "-q", "-p", "no:cacheprovider"],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    if r.returncode != 1:
        return f"{name}: no pin failed (exit {r.returncode})\n{r.stdout[-1500:]}"
    return None


def test_pins_catch_every_mutant(tmp_path):
    workers = max(1, min(8, (os.cpu_count() or 2) // 2))
    with ThreadPoolExecutor(max_workers=workers) as ex:
        results = list(ex.map(lambda m: _run_mutant(tmp_path, *m), MUTANTS))
    missed = [r for r in results if r]
    assert not missed, "\n".join(missed)
