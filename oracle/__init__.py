"""ctypes front end of the CPU oracle (``moe_oracle.c``).

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the bench's CPU-baseline leg
import this module; the product package never does. The oracle is a plain, slow C
restatement of the MoE layer forward (Comet: Fine-grained Computation-communication
Overlapping for Mixture-of-Experts, §2.1 "MoE Structure"; the tile reorganisation of
§2.2.1 and §3.1.2). Every function here only marshals numpy arrays into the C entry
points; no arithmetic of the method lives in Python.

Arrays of bf16 values are passed as ``numpy.uint16`` bit patterns.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from pathlib import Path

import numpy as np

_HERE = Path(__file__).resolve().parent
_SRC = _HERE / "moe_oracle.c"
_LIB = _HERE / "liboracle.so"

ACT_SWIGLU, ACT_GELU_TANH, ACT_RELU, ACT_IDENTITY = 0, 1, 2, 3
GATE_SOFTMAX_TOPK, GATE_SOFTMAX_ALL, GATE_SELECT_BIAS = 0, 1, 2

# Portable flags: the library may be built on one host and run on another.
CFLAGS = ["-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off", "-fopenmp"]


def build(force: bool = False, src: Path | None = None, out: Path | None = None) -> Path:
    """Compile the oracle into a shared library (gcc) and return its path."""
    src = Path(src) if src is not None else _SRC
    out = Path(out) if out is not None else _LIB
    if force or not out.exists() or out.stat().st_mtime < src.stat().st_mtime:
        tmp = out.with_suffix(f".tmp{os.getpid()}.so")
        subprocess.run(["gcc", *CFLAGS, "-o", str(tmp), str(src), "-lm"], check=True)
        os.replace(tmp, out)
    return out


_lib_cache: dict[str, ctypes.CDLL] = {}


def load(path: Path | None = None) -> ctypes.CDLL:
    """Load (building first if needed) the oracle library; cached per path."""
    p = str(build() if path is None else path)
    if p in _lib_cache:
        return _lib_cache[p]
    lib = ctypes.CDLL(p)
    i32, i64, vp = ctypes.c_int, ctypes.c_int64, ctypes.c_void_p
    lib.oracle_round_to_bf16.argtypes = [ctypes.c_double]
    lib.oracle_round_to_bf16.restype = ctypes.c_double
    lib.oracle_router_logits.argtypes = [i32, i32, i32, vp, vp, vp, vp]
    lib.oracle_router_logits.restype = None
    lib.oracle_topk_gates.argtypes = [i32, i32, i32, i32, vp, vp, vp]
    lib.oracle_topk_gates.restype = i32
    lib.oracle_topk_gates_bias.argtypes = [i32, i32, i32, i32, vp, vp, vp, vp]
    lib.oracle_topk_gates_bias.restype = i32
    lib.oracle_shared_tokens.argtypes = [i32, i32, i32, vp, vp, vp, vp, i32, vp, vp]
    lib.oracle_shared_tokens.restype = i32
    lib.oracle_dispatch.argtypes = [i32, i32, i32, i32, vp, vp, vp, vp, vp, i64, vp, vp, vp, vp, i64]
    lib.oracle_dispatch.restype = i32
    lib.oracle_expert_ffn_row.argtypes = [i32, i32, i32, i32, vp, vp, vp, vp]
    lib.oracle_expert_ffn_row.restype = None
    lib.oracle_combine.argtypes = [i32, i32, i32, vp, vp, vp]
    lib.oracle_combine.restype = None
    lib.oracle_moe_forward.argtypes = [i32] * 9 + [vp] * 8
    lib.oracle_moe_forward.restype = i32
    lib.oracle_moe_tokens.argtypes = [i32] * 8 + [vp] * 5 + [i32, vp, vp, vp, vp]
    lib.oracle_moe_tokens.restype = i32
    lib.oracle_e4m3_encode.argtypes = [ctypes.c_float]
    lib.oracle_e4m3_encode.restype = ctypes.c_uint8
    lib.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
    lib.oracle_e4m3_decode.restype = ctypes.c_double
    lib.oracle_e4m3_encode_n.argtypes = [i64, vp, vp]
    lib.oracle_e4m3_encode_n.restype = None
    lib.oracle_e4m3_decode_n.argtypes = [i64, vp, vp]
    lib.oracle_e4m3_decode_n.restype = None
    lib.oracle_quant_rows_fp8.argtypes = [i32, i32, vp, vp, vp]
    lib.oracle_quant_rows_fp8.restype = None
    lib.oracle_quant_cols_fp8.argtypes = [i32, i32, i32, vp, vp, vp]
    lib.oracle_quant_cols_fp8.restype = None
    lib.oracle_moe_tokens_fp8.argtypes = [i32] * 7 + [vp] * 7 + [i32, vp, vp, vp, vp]
    lib.oracle_moe_tokens_fp8.restype = i32
    lib.oracle_e8m0_decode.argtypes = [ctypes.c_uint8]
    lib.oracle_e8m0_decode.restype = ctypes.c_double
    lib.oracle_mx_quant_rows_f32.argtypes = [i32, i32, vp, vp, vp]
    lib.oracle_mx_quant_rows_f32.restype = i32
    lib.oracle_mx_quant_rows.argtypes = [i32, i32, vp, vp, vp]
    lib.oracle_mx_quant_rows.restype = i32
    lib.oracle_mx_quant_cols.argtypes = [i32, i32, i32, vp, vp, vp]
    lib.oracle_mx_quant_cols.restype = i32
    lib.oracle_moe_tokens_mx.argtypes = [i32] * 7 + [vp] * 7 + [i32, vp, vp, vp, vp]
    lib.oracle_moe_tokens_mx.restype = i32
    lib.oracle_moe_backward.argtypes = [i32] * 7 + [vp] * 11
    lib.oracle_moe_backward.restype = i32
    lib.oracle_moe_backward_dx_tokens.argtypes = [i32] * 7 + [vp] * 6 + [i32, vp, vp]
    lib.oracle_moe_backward_dx_tokens.restype = i32
    _lib_cache[p] = lib
    return lib


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _u16(a):
    a = np.ascontiguousarray(a)
    assert a.dtype == np.uint16, a.dtype
    return a


def round_to_bf16(v: float, lib=None) -> float:
    return (lib or load()).oracle_round_to_bf16(float(v))


def router_logits(x, Wg, bias=None, lib=None):
    """fp32 logits [T,E] (sequential h-ascending sum; see moe_oracle.c)."""
    lib = lib or load()
    x, Wg = _u16(x), _u16(Wg)
    T, H = x.shape
    H2, E = Wg.shape
    assert H == H2
    b = None if bias is None else np.ascontiguousarray(bias, dtype=np.float32)
    out = np.empty((T, E), np.float32)
    lib.oracle_router_logits(T, H, E, _p(x), _p(Wg), _p(b), _p(out))
    return out


def topk_gates(logits, k, gate=GATE_SOFTMAX_TOPK, lib=None, bias=None):
    """bias: used by GATE_SELECT_BIAS only (the logits then exclude it)."""
    lib = lib or load()
    logits = np.ascontiguousarray(logits, dtype=np.float32)
    T, E = logits.shape
    idx = np.empty((T, k), np.int32)
    w = np.empty((T, k), np.float64)
    b = None if bias is None else np.ascontiguousarray(bias, dtype=np.float32)
    rc = lib.oracle_topk_gates_bias(T, E, k, gate, _p(logits), _p(b), _p(idx), _p(w))
    if rc:
        raise ValueError(f"oracle_topk_gates rc={rc}")
    return idx, w


def padded_rows_max(T, E, k, m_tile=128):
    return T * k + E * (m_tile - 1)


def dispatch(idx, E, m_tile=128, lib=None):
    """Counting sort of routed pairs into expert-contiguous, m_tile-padded rows."""
    lib = lib or load()
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    T, k = idx.shape
    glen = padded_rows_max(T, E, k, m_tile)
    tcap = glen // m_tile + E
    counts = np.empty(E, np.int32)
    offsets = np.empty(E + 1, np.int32)
    poff = np.empty(E + 1, np.int32)
    gather_idx = np.empty(glen, np.int32)
    inv_pos = np.empty((T, k), np.int32)
    te = np.empty(tcap, np.int32)
    tr = np.empty(tcap, np.int32)
    tn = np.empty(tcap, np.int32)
    nt = lib.oracle_dispatch(T, E, k, m_tile, _p(idx), _p(counts), _p(offsets), _p(poff),
                             _p(gather_idx), glen, _p(inv_pos), _p(te), _p(tr), _p(tn), tcap)
    if nt < 0:
        raise ValueError(f"oracle_dispatch rc={nt}")
    return dict(counts=counts, offsets=offsets, padded_offsets=poff, gather_idx=gather_idx,
                inv_pos=inv_pos, tile_expert=te[:nt].copy(), tile_row0=tr[:nt].copy(),
                tile_nvalid=tn[:nt].copy(), num_tiles=nt)


def expert_ffn_row(xrow, W1e, W2e, act=ACT_SWIGLU, round_a_bf16=False, lib=None):
    lib = lib or load()
    xrow, W1e, W2e = _u16(xrow), _u16(W1e), _u16(W2e)
    H = xrow.shape[0]
    F, H2 = W2e.shape
    assert H2 == H
    y = np.empty(H, np.float64)
    lib.oracle_expert_ffn_row(H, F, act, int(round_a_bf16), _p(xrow), _p(W1e), _p(W2e), _p(y))
    return y


def combine(ys, inv_pos, lib=None):
    """out[t] = sum_j ys[inv_pos[t, j]] (fp64; ys are bf16 rows already gate-scaled)."""
    lib = lib or load()
    ys = _u16(ys)
    inv_pos = np.ascontiguousarray(inv_pos, dtype=np.int32)
    T, k = inv_pos.shape
    H = ys.shape[1]
    out = np.empty((T, H), np.float64)
    lib.oracle_combine(T, H, k, _p(ys), _p(inv_pos), _p(out))
    return out


def _ffn_dims(W1, W2, act):
    E, H, c = W1.shape
    E2, F, H2 = W2.shape
    assert E == E2 and H == H2
    assert c == (2 * F if act == ACT_SWIGLU else F), (c, F, act)
    return E, H, F


def moe_forward(x, Wg, bias, W1, W2, k, act=ACT_SWIGLU, gate=GATE_SOFTMAX_TOPK, m_tile=128,
                round_a_bf16=False, lib=None):
    """Whole layer (route -> dispatch -> experts -> combine). Returns (out f64 [T,H], idx, w)."""
    lib = lib or load()
    x, Wg, W1, W2 = _u16(x), _u16(Wg), _u16(W1), _u16(W2)
    T, H = x.shape
    E, H1, F = _ffn_dims(W1, W2, act)
    assert H1 == H and Wg.shape == (H, E)
    b = None if bias is None else np.ascontiguousarray(bias, dtype=np.float32)
    out = np.empty((T, H), np.float64)
    idx = np.empty((T, k), np.int32)
    w = np.empty((T, k), np.float64)
    rc = lib.oracle_moe_forward(T, H, F, E, k, act, gate, m_tile, int(round_a_bf16), _p(x), _p(Wg),
                                _p(b), _p(W1), _p(W2), _p(out), _p(idx), _p(w))
    if rc:
        raise ValueError(f"oracle_moe_forward rc={rc}")
    return out, idx, w


def moe_tokens(x, Wg, bias, W1, W2, k, tokens, act=ACT_SWIGLU, gate=GATE_SOFTMAX_TOPK,
               round_a_bf16=False, lib=None):
    """Layer output for selected tokens straight from the per-token definition."""
    lib = lib or load()
    x, Wg, W1, W2 = _u16(x), _u16(Wg), _u16(W1), _u16(W2)
    T, H = x.shape
    E, H1, F = _ffn_dims(W1, W2, act)
    assert H1 == H and Wg.shape == (H, E)
    tokens = np.ascontiguousarray(tokens, dtype=np.int32)
    n = tokens.shape[0]
    b = None if bias is None else np.ascontiguousarray(bias, dtype=np.float32)
    out = np.empty((n, H), np.float64)
    idx = np.empty((n, k), np.int32)
    w = np.empty((n, k), np.float64)
    rc = lib.oracle_moe_tokens(T, H, F, E, k, act, gate, int(round_a_bf16), _p(x), _p(Wg), _p(b),
                               _p(W1), _p(W2), n, _p(tokens), _p(out), _p(idx), _p(w))
    if rc:
        raise ValueError(f"oracle_moe_tokens rc={rc}")
    return out, idx, w


def shared_tokens(x, W1s, W2s, w_sg, tokens, lib=None):
    """Shared-expert term g_t * FFN_s(x_t) for the listed tokens (fp64 [ntok, H]).
    W1s [H, 2Fs], W2s [Fs, H], w_sg [H] or None (gate 1)."""
    lib = lib or load()
    x, W1s, W2s = _u16(x), _u16(W1s), _u16(W2s)
    wg = None if w_sg is None else _u16(w_sg)
    T, H = x.shape
    Fs = W2s.shape[0]
    assert W1s.shape == (H, 2 * Fs) and W2s.shape == (Fs, H)
    tokens = np.ascontiguousarray(tokens, dtype=np.int32)
    out = np.empty((tokens.size, H), np.float64)
    rc = lib.oracle_shared_tokens(T, H, Fs, _p(x), _p(W1s), _p(W2s), _p(wg), tokens.size,
                                  _p(tokens), _p(out))
    if rc:
        raise ValueError(f"oracle_shared_tokens rc={rc}")
    return out


# ---------------------------------------------------------------------------------------
# FP8 (e4m3) experts: a precision variant outside the pages (see moe_oracle.c for the
# reading: per-row scales of x and h, per-output-column scales of W1 and W2)
# ---------------------------------------------------------------------------------------

def e4m3_encode(v, lib=None):
    """float32 values -> e4m3 codes (uint8), nearest with ties to even, saturating."""
    lib = lib or load()
    v = np.ascontiguousarray(v, dtype=np.float32)
    out = np.empty(v.shape, np.uint8)
    lib.oracle_e4m3_encode_n(v.size, _p(v), _p(out))
    return out


def e4m3_decode(c, lib=None):
    """e4m3 codes (uint8) -> their values (fp64; NaN for the NaN codes)."""
    lib = lib or load()
    c = np.ascontiguousarray(c, dtype=np.uint8)
    out = np.empty(c.shape, np.float64)
    lib.oracle_e4m3_decode_n(c.size, _p(c), _p(out))
    return out


def quant_rows_fp8(src, lib=None):
    """bf16 bit patterns [rows, cols] -> (codes [rows, cols] uint8, scales [rows] fp32)."""
    lib = lib or load()
    src = _u16(src)
    rows, cols = src.shape
    q = np.empty((rows, cols), np.uint8)
    s = np.empty(rows, np.float32)
    lib.oracle_quant_rows_fp8(rows, cols, _p(src), _p(q), _p(s))
    return q, s


def quant_cols_fp8(W, lib=None):
    """Expert weights, bf16 bit patterns [E, K, N] -> (codes [E, N, K] uint8, scales [E, N])."""
    lib = lib or load()
    W = _u16(W)
    E, K, N = W.shape
    q = np.empty((E, N, K), np.uint8)
    s = np.empty((E, N), np.float32)
    lib.oracle_quant_cols_fp8(E, K, N, _p(W), _p(q), _p(s))
    return q, s


def moe_tokens_fp8(x, Wg, bias, W1q, s1, W2q, s2, k, tokens, act=ACT_SWIGLU,
                   gate=GATE_SOFTMAX_TOPK, lib=None):
    """Layer output with e4m3 experts for the listed tokens (fp64 [ntok, H]), plus the
    routing. W1q [E, w1_cols, H], s1 [E, w1_cols], W2q [E, H, F], s2 [E, H]."""
    lib = lib or load()
    x, Wg = _u16(x), _u16(Wg)
    T, H = x.shape
    E = Wg.shape[1]
    W1q = np.ascontiguousarray(W1q, dtype=np.uint8)
    W2q = np.ascontiguousarray(W2q, dtype=np.uint8)
    s1 = np.ascontiguousarray(s1, dtype=np.float32)
    s2 = np.ascontiguousarray(s2, dtype=np.float32)
    F = W2q.shape[2]
    w1_cols = 2 * F if act == ACT_SWIGLU else F
    assert W1q.shape == (E, w1_cols, H) and s1.shape == (E, w1_cols)
    assert W2q.shape == (E, H, F) and s2.shape == (E, H)
    tokens = np.ascontiguousarray(tokens, dtype=np.int32)
    n = tokens.shape[0]
    b = None if bias is None else np.ascontiguousarray(bias, dtype=np.float32)
    out = np.empty((n, H), np.float64)
    idx = np.empty((n, k), np.int32)
    w = np.empty((n, k), np.float64)
    rc = lib.oracle_moe_tokens_fp8(T, H, F, E, k, act, gate, _p(x), _p(Wg), _p(b), _p(W1q),
                                   _p(s1), _p(W2q), _p(s2), n, _p(tokens), _p(out), _p(idx), _p(w))
    if rc:
        raise ValueError(f"oracle_moe_tokens_fp8 rc={rc}")
    return out, idx, w


# ---------------------------------------------------------------------------------------
# Block-scaled FP8 (MX form: e4m3 codes, one e8m0 power-of-two scale per 32 values along K;
# see moe_oracle.c for the reading). Oracle only: no CUDA path for this form yet.
# ---------------------------------------------------------------------------------------

def e8m0_decode(b, lib=None):
    """e8m0 scale byte -> 2^(b - 127) (NaN for 255)."""
    lib = lib or load()
    return float(lib.oracle_e8m0_decode(int(b)))


def mx_quant_rows_f32(v, lib=None):
    """float32 values [rows, cols] (cols % 32 == 0) -> (codes [rows, cols] uint8, scale
    bytes [rows, cols / 32] uint8)."""
    lib = lib or load()
    v = np.ascontiguousarray(v, dtype=np.float32)
    rows, cols = v.shape
    q = np.empty((rows, cols), np.uint8)
    s = np.empty((rows, cols // 32), np.uint8)
    if lib.oracle_mx_quant_rows_f32(rows, cols, _p(v), _p(q), _p(s)):
        raise ValueError("cols must be a multiple of 32")
    return q, s


def mx_quant_rows(src, lib=None):
    """bf16 bit patterns [rows, cols] -> (codes [rows, cols], scale bytes [rows, cols / 32])."""
    lib = lib or load()
    src = _u16(src)
    rows, cols = src.shape
    q = np.empty((rows, cols), np.uint8)
    s = np.empty((rows, cols // 32), np.uint8)
    if lib.oracle_mx_quant_rows(rows, cols, _p(src), _p(q), _p(s)):
        raise ValueError("cols must be a multiple of 32")
    return q, s


def mx_quant_cols(W, lib=None):
    """Expert weights, bf16 bit patterns [E, K, N] -> (codes [E, N, K], scale bytes
    [E, N, K / 32]): per output column, blocks of 32 along K."""
    lib = lib or load()
    W = _u16(W)
    E, K, N = W.shape
    q = np.empty((E, N, K), np.uint8)
    s = np.empty((E, N, K // 32), np.uint8)
    if lib.oracle_mx_quant_cols(E, K, N, _p(W), _p(q), _p(s)):
        raise ValueError("K must be a multiple of 32")
    return q, s


def moe_tokens_mx(x, Wg, bias, W1q, W1s, W2q, W2s, k, tokens, act=ACT_SWIGLU,
                  gate=GATE_SOFTMAX_TOPK, lib=None):
    """Layer output with MX experts for the listed tokens (fp64 [ntok, H]), plus the routing.
    W1q [E, w1_cols, H], W1s [E, w1_cols, H / 32], W2q [E, H, F], W2s [E, H, F / 32]."""
    lib = lib or load()
    x, Wg = _u16(x), _u16(Wg)
    T, H = x.shape
    E = Wg.shape[1]
    W1q = np.ascontiguousarray(W1q, dtype=np.uint8)
    W2q = np.ascontiguousarray(W2q, dtype=np.uint8)
    W1s = np.ascontiguousarray(W1s, dtype=np.uint8)
    W2s = np.ascontiguousarray(W2s, dtype=np.uint8)
    F = W2q.shape[2]
    w1_cols = 2 * F if act == ACT_SWIGLU else F
    assert W1q.shape == (E, w1_cols, H) and W1s.shape == (E, w1_cols, H // 32)
    assert W2q.shape == (E, H, F) and W2s.shape == (E, H, F // 32)
    tokens = np.ascontiguousarray(tokens, dtype=np.int32)
    n = tokens.shape[0]
    b = None if bias is None else np.ascontiguousarray(bias, dtype=np.float32)
    out = np.empty((n, H), np.float64)
    idx = np.empty((n, k), np.int32)
    w = np.empty((n, k), np.float64)
    rc = lib.oracle_moe_tokens_mx(T, H, F, E, k, act, gate, _p(x), _p(Wg), _p(b), _p(W1q),
                                  _p(W1s), _p(W2q), _p(W2s), n, _p(tokens), _p(out), _p(idx), _p(w))
    if rc:
        raise ValueError(f"oracle_moe_tokens_mx rc={rc}")
    return out, idx, w


# ---------------------------------------------------------------------------------------
# Backward pass (training; beyond the pages): gradients of the layer for a given dL/dout
# ---------------------------------------------------------------------------------------

def moe_backward(x, Wg, bias, W1, W2, dy, k, act=ACT_SWIGLU, gate=GATE_SOFTMAX_TOPK, lib=None):
    """All gradients (fp64): dict(dx [T,H], dWg [H,E], dbias [E], dW1 [E,H,w1c], dW2 [E,F,H])."""
    lib = lib or load()
    x, Wg, W1, W2, dy = _u16(x), _u16(Wg), _u16(W1), _u16(W2), _u16(dy)
    T, H = x.shape
    E, H1, F = _ffn_dims(W1, W2, act)
    assert H1 == H and Wg.shape == (H, E) and dy.shape == (T, H)
    b = None if bias is None else np.ascontiguousarray(bias, dtype=np.float32)
    g = dict(dx=np.empty((T, H)), dWg=np.empty((H, E)), dbias=np.empty(E),
             dW1=np.empty(W1.shape), dW2=np.empty(W2.shape))
    rc = lib.oracle_moe_backward(T, H, F, E, k, act, gate, _p(x), _p(Wg), _p(b), _p(W1), _p(W2),
                                 _p(dy), _p(g["dx"]), _p(g["dWg"]), _p(g["dbias"]), _p(g["dW1"]),
                                 _p(g["dW2"]))
    if rc:
        raise ValueError(f"oracle_moe_backward rc={rc}")
    return g


def moe_backward_dx_tokens(x, Wg, bias, W1, W2, dy, k, tokens, act=ACT_SWIGLU,
                           gate=GATE_SOFTMAX_TOPK, lib=None):
    """Input gradient dx (fp64 [ntok, H]) of the listed tokens only."""
    lib = lib or load()
    x, Wg, W1, W2, dy = _u16(x), _u16(Wg), _u16(W1), _u16(W2), _u16(dy)
    T, H = x.shape
    E, _, F = _ffn_dims(W1, W2, act)
    tokens = np.ascontiguousarray(tokens, dtype=np.int32)
    b = None if bias is None else np.ascontiguousarray(bias, dtype=np.float32)
    out = np.empty((tokens.size, H))
    rc = lib.oracle_moe_backward_dx_tokens(T, H, F, E, k, act, gate, _p(x), _p(Wg), _p(b), _p(W1),
                                           _p(W2), _p(dy), tokens.size, _p(tokens), _p(out))
    if rc:
        raise ValueError(f"oracle_moe_backward_dx_tokens rc={rc}")
    return out
