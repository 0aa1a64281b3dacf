"""ctypes binding of libmoe_b200.so (include/moe.h). Argument marshalling only.

Every function takes torch tensors (or None for optional pointers), checks dtype, device
and contiguity, passes ``data_ptr()`` and the current CUDA stream to the C entry point of
the same name, and raises ``MoeError`` on a non-OK status. No computation of the layer
happens here.
"""
from __future__ import annotations

import ctypes
import threading
from pathlib import Path

import torch

from .build import LIB_PATH

ACT_SWIGLU, ACT_GELU_TANH, ACT_RELU, ACT_IDENTITY = 0, 1, 2, 3
GATE_SOFTMAX_TOPK, GATE_SOFTMAX_ALL, GATE_SELECT_BIAS = 0, 1, 2
MOE_NUM_STAGE_EVENTS = 6
M_TILE = 128

STATUS_NAMES = {
    0: "MOE_OK",
    -1: "MOE_ERR_INVALID_ARG",
    -2: "MOE_ERR_UNSUPPORTED",
    -3: "MOE_ERR_WORKSPACE",
    -4: "MOE_ERR_CUDA",
    -5: "MOE_ERR_DEVICE_TIMEOUT",
    -6: "MOE_ERR_DEVICE_BAD_INDEX",
}


class MoeError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} failed: {STATUS_NAMES.get(status, status)}")
        self.status = status


class Problem(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int32), ("H", ctypes.c_int32), ("F", ctypes.c_int32),
                ("E", ctypes.c_int32), ("top_k", ctypes.c_int32), ("act", ctypes.c_int32),
                ("gate", ctypes.c_int32), ("m_tile", ctypes.c_int32)]

    @classmethod
    def make(cls, T, H, F, E, top_k, act=ACT_SWIGLU, gate=GATE_SOFTMAX_TOPK, m_tile=M_TILE):
        return cls(T, H, F, E, top_k, act, gate, m_tile)

    @classmethod
    def from_config(cls, cfg):
        return cls.make(cfg.T, cfg.H, cfg.F, cfg.E, cfg.k, cfg.act, cfg.gate)


class SharedExpert(ctypes.Structure):
    """moe_shared_expert: width F_s and device pointers of W1s [H, 2F_s], W2s [F_s, H], w_sg [H]."""
    _fields_ = [("F_s", ctypes.c_int32), ("W1s", ctypes.c_void_p), ("W2s", ctypes.c_void_p),
                ("w_sg", ctypes.c_void_p)]


EP_MAX_WORLD = 8
EP_MAX_LOCAL = 4
EP_BUFFERS = ("counts", "flags", "recv_rows", "recv_gate", "recv_origin", "arrive", "back",
              "back_cnt")


class EpRank(ctypes.Structure):
    """moe_ep_rank: one rank of moe_ep_layer_forward (device pointers; buf[b][d] is rank d's
    exchange buffer b as this GPU addresses it, b in the order of EP_BUFFERS)."""
    _fields_ = [("p", Problem), ("world", ctypes.c_int32), ("rank", ctypes.c_int32),
                ("epoch", ctypes.c_int32), ("x", ctypes.c_void_p), ("Wg", ctypes.c_void_p),
                ("bias", ctypes.c_void_p), ("W1", ctypes.c_void_p), ("W2", ctypes.c_void_p),
                ("out", ctypes.c_void_p), ("topk_idx", ctypes.c_void_p),
                ("topk_w", ctypes.c_void_p), ("ws", ctypes.c_void_p),
                ("ws_bytes", ctypes.c_size_t),
                ("buf", (ctypes.c_void_p * EP_MAX_WORLD) * len(EP_BUFFERS))]


_lock = threading.Lock()
_lib = None


def library_path() -> Path:
    return LIB_PATH


def library() -> ctypes.CDLL:
    """Load libmoe_b200.so. Raises if it has not been built: there is no fallback path."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not LIB_PATH.exists():
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with `python -c 'import __graft_entry__ as g; "
                f"g.build()'` (nvcc, sm_100a). There is no CPU fallback.")
        lib = ctypes.CDLL(str(LIB_PATH))
        vp, sz, i32, i64 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int, ctypes.c_int64
        P = ctypes.POINTER(Problem)
        sig = {
            "moe_workspace_size": ([P], sz),
            "moe_forward_launches": ([P], i32),
            "moe_route_uses_filter": ([P], i32),
            "moe_padded_rows_max": ([P], i64),
            "moe_route": ([P, vp, vp, vp, vp, vp, vp, sz, vp], i32),
            "moe_route_noalloc": ([P, vp, vp, vp, vp, vp, vp], i32),
            "moe_dispatch": ([P, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp], i32),
            "moe_forward": ([P, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp], i32),
            "moe_forward_staged": ([P, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp,
                                    ctypes.POINTER(vp), i32], i32),
            "moe_forward_host": ([P, vp, vp, vp, vp, vp, vp, vp, sz, vp], i32),
            "moe_forward_host_batches": ([P, i32, vp, vp, vp, vp, vp, vp, vp, sz, vp], i32),
            "moe_workspace_size_shared": ([P, i32], sz),
            "moe_forward_shared": ([P, vp, vp, vp, vp, vp, ctypes.POINTER(SharedExpert), vp, vp,
                                    vp, vp, sz, vp], i32),
            "moe_workspace_size_fp8": ([P], sz),
            "moe_quantize_experts_fp8": ([P, vp, vp, vp, vp, vp, vp, vp], i32),
            "moe_quantize_rows_fp8": ([vp, i64, i32, vp, vp, vp], i32),
            "moe_forward_fp8": ([P, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp], i32),
            "moe_forward_fp8_staged": ([P, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp,
                                        ctypes.POINTER(vp), i32], i32),
            "moe_experts_forward": ([P] + [vp] * 7 + [sz, vp], i32),
            "moe_experts_forward_n": ([P] + [vp] * 8 + [sz, vp], i32),
            "moe_ep_publish_counts": ([P, i32, i32, vp, vp, vp], i32),
            "moe_ep_scatter": ([P, i32, i32] + [vp] * 11 + [i64, vp, vp, sz, vp], i32),
            "moe_ep_return": ([i32, i32, vp, vp, vp, i64, vp, i64, vp, vp], i32),
            "moe_backward_workspace_size": ([P], sz),
            "moe_backward": ([P] + [vp] * 12 + [sz, vp], i32),
            "moe_combine": ([P, vp, i64, vp, vp, vp, sz, vp], i32),
            "moe_get_device_status": ([vp, vp], i32),
            "moe_status_string": ([i32], ctypes.c_char_p),
            "moe_set_wait_timeout_ns": ([i64], i64),
            "moe_set_gemm_mode": ([i32], i32),
            "moe_set_fault_injection": ([i32], i32),
            "moe_set_schedule_trace": ([vp, i64], i32),
            "moe_set_router_mode": ([i32], i32),
            "moe_set_work_order": ([i32], i32),
            "moe_set_whole_layer_launch": ([i32], i32),
            "moe_ep_buffer_sizes": ([P, i32, ctypes.POINTER(ctypes.c_int64)], i32),
            "moe_ep_workspace_size": ([P, i32], sz),
            "moe_ep_layer_forward": ([ctypes.POINTER(EpRank), i32, vp], i32),
        }
        for name, (args, res) in sig.items():
            f = getattr(lib, name)
            f.argtypes = args
            f.restype = res
        _lib = lib
        return lib


# ---------------------------------------------------------------------------------------
# marshalling helpers
# ---------------------------------------------------------------------------------------

def _ptr(t, dtype=None, name="tensor", cuda=True):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if cuda and not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not cuda and t.is_cuda:
        raise ValueError(f"{name} must be a host tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def _check(fn, rc):
    if rc != 0:
        raise MoeError(fn, rc)


def _ws(ws):
    return _ptr(ws, torch.uint8, "ws"), ctypes.c_size_t(ws.numel())


# ---------------------------------------------------------------------------------------
# entry points
# ---------------------------------------------------------------------------------------

def moe_workspace_size(p: Problem) -> int:
    return int(library().moe_workspace_size(ctypes.byref(p)))


def moe_forward_launches(p: Problem) -> int:
    """Kernels one moe_forward call on p launches under the current GEMM and router modes."""
    return int(library().moe_forward_launches(ctypes.byref(p)))


def moe_route_uses_filter(p: Problem) -> bool:
    """Whether the router on p takes the filter variant under the current router mode."""
    rc = int(library().moe_route_uses_filter(ctypes.byref(p)))
    if rc < 0:
        raise ValueError("moe_route_uses_filter: invalid problem")
    return rc == 1


def moe_padded_rows_max(p: Problem) -> int:
    return int(library().moe_padded_rows_max(ctypes.byref(p)))


def moe_route(p, x, Wg, bias, topk_idx, topk_w, ws, stream=None):
    bf, i32, f32 = torch.bfloat16, torch.int32, torch.float32
    w, n = _ws(ws)
    rc = library().moe_route(ctypes.byref(p), _ptr(x, bf, "x"), _ptr(Wg, bf, "Wg"),
                             _ptr(bias, f32, "bias"), _ptr(topk_idx, i32, "topk_idx"),
                             _ptr(topk_w, f32, "topk_w"), w, n, _stream(stream))
    _check("moe_route", rc)


def moe_route_noalloc(p, x, Wg, bias, topk_idx, topk_w, stream=None):
    """moe_route without a workspace (the library's fixed scratch array holds the logits).
    For callers that cannot allocate device memory; see include/moe.h for the size limit
    and the rule that overlapping calls race."""
    bf, i32, f32 = torch.bfloat16, torch.int32, torch.float32
    rc = library().moe_route_noalloc(ctypes.byref(p), _ptr(x, bf, "x"), _ptr(Wg, bf, "Wg"),
                                     _ptr(bias, f32, "bias"), _ptr(topk_idx, i32, "topk_idx"),
                                     _ptr(topk_w, f32, "topk_w"), _stream(stream))
    _check("moe_route_noalloc", rc)


def moe_dispatch(p, topk_idx, counts, offsets, padded_offsets, gather_idx, inv_pos, ws,
                 x_perm=None, x=None, stream=None):
    bf, i32 = torch.bfloat16, torch.int32
    w, n = _ws(ws)
    rc = library().moe_dispatch(ctypes.byref(p), _ptr(topk_idx, i32, "topk_idx"),
                                _ptr(counts, i32, "counts"), _ptr(offsets, i32, "offsets"),
                                _ptr(padded_offsets, i32, "padded_offsets"),
                                _ptr(gather_idx, i32, "gather_idx"), _ptr(inv_pos, i32, "inv_pos"),
                                _ptr(x_perm, bf, "x_perm"), _ptr(x, bf, "x"), w, n, _stream(stream))
    _check("moe_dispatch", rc)


def moe_forward(p, x, Wg, bias, W1, W2, out, ws, topk_idx_out=None, topk_w_out=None, stream=None):
    bf = torch.bfloat16
    w, n = _ws(ws)
    rc = library().moe_forward(ctypes.byref(p), _ptr(x, bf, "x"), _ptr(Wg, bf, "Wg"),
                               _ptr(bias, torch.float32, "bias"), _ptr(W1, bf, "W1"),
                               _ptr(W2, bf, "W2"), _ptr(out, bf, "out"),
                               _ptr(topk_idx_out, torch.int32, "topk_idx_out"),
                               _ptr(topk_w_out, torch.float32, "topk_w_out"), w, n, _stream(stream))
    _check("moe_forward", rc)


def moe_forward_staged(p, x, Wg, bias, W1, W2, out, ws, events, topk_idx_out=None,
                       topk_w_out=None, stream=None):
    """``events``: MOE_NUM_STAGE_EVENTS torch.cuda.Event(enable_timing=True) objects."""
    bf = torch.bfloat16
    w, n = _ws(ws)
    if len(events) != MOE_NUM_STAGE_EVENTS:
        raise ValueError(f"need {MOE_NUM_STAGE_EVENTS} events")
    for ev in events:
        if ev.cuda_event == 0:   # torch creates the CUDA event lazily, on its first record
            ev.record()
    arr = (ctypes.c_void_p * MOE_NUM_STAGE_EVENTS)(*[ctypes.c_void_p(e.cuda_event) for e in events])
    rc = library().moe_forward_staged(ctypes.byref(p), _ptr(x, bf, "x"), _ptr(Wg, bf, "Wg"),
                                      _ptr(bias, torch.float32, "bias"), _ptr(W1, bf, "W1"),
                                      _ptr(W2, bf, "W2"), _ptr(out, bf, "out"),
                                      _ptr(topk_idx_out, torch.int32, "topk_idx_out"),
                                      _ptr(topk_w_out, torch.float32, "topk_w_out"), w, n,
                                      _stream(stream), arr, MOE_NUM_STAGE_EVENTS)
    _check("moe_forward_staged", rc)


def moe_forward_host(p, x_host, Wg, bias, W1, W2, out_host, ws, stream=None):
    """Activations on the host (pinned for async copies), weights on the device."""
    bf = torch.bfloat16
    w, n = _ws(ws)
    rc = library().moe_forward_host(ctypes.byref(p), _ptr(x_host, bf, "x_host", cuda=False),
                                    _ptr(Wg, bf, "Wg"), _ptr(bias, torch.float32, "bias"),
                                    _ptr(W1, bf, "W1"), _ptr(W2, bf, "W2"),
                                    _ptr(out_host, bf, "out_host", cuda=False), w, n,
                                    _stream(stream))
    _check("moe_forward_host", rc)


def moe_forward_host_batches(p, xs_host, Wg, bias, W1, W2, outs_host, ws, stream=None):
    """A stream of host batches (lists of pinned [T, H] bf16 tensors): each batch's copies in
    and out overlap the neighbouring batches' compute. Returns when the last output landed."""
    bf = torch.bfloat16
    n = len(xs_host)
    if len(outs_host) != n:
        raise ValueError("xs_host and outs_host differ in length")
    xa = (ctypes.c_void_p * max(n, 1))(*[_ptr(x, bf, "x_host", cuda=False) for x in xs_host])
    oa = (ctypes.c_void_p * max(n, 1))(*[_ptr(o, bf, "out_host", cuda=False) for o in outs_host])
    w, nb = _ws(ws)
    rc = library().moe_forward_host_batches(ctypes.byref(p), n, ctypes.cast(xa, ctypes.c_void_p),
                                            _ptr(Wg, bf, "Wg"), _ptr(bias, torch.float32, "bias"),
                                            _ptr(W1, bf, "W1"), _ptr(W2, bf, "W2"),
                                            ctypes.cast(oa, ctypes.c_void_p), w, nb,
                                            _stream(stream))
    _check("moe_forward_host_batches", rc)


def moe_workspace_size_shared(p: Problem, F_s: int) -> int:
    return int(library().moe_workspace_size_shared(ctypes.byref(p), int(F_s)))


def moe_forward_shared(p, x, Wg, bias, W1, W2, W1s, W2s, w_sg, out, ws, topk_idx_out=None,
                       topk_w_out=None, stream=None):
    """moe_forward plus a shared expert: W1s [H, 2F_s], W2s [F_s, H], w_sg [H] or None."""
    bf = torch.bfloat16
    sh = SharedExpert(int(W2s.shape[0]), _ptr(W1s, bf, "W1s"), _ptr(W2s, bf, "W2s"),
                      _ptr(w_sg, bf, "w_sg"))
    w, n = _ws(ws)
    rc = library().moe_forward_shared(ctypes.byref(p), _ptr(x, bf, "x"), _ptr(Wg, bf, "Wg"),
                                      _ptr(bias, torch.float32, "bias"), _ptr(W1, bf, "W1"),
                                      _ptr(W2, bf, "W2"), ctypes.byref(sh), _ptr(out, bf, "out"),
                                      _ptr(topk_idx_out, torch.int32, "topk_idx_out"),
                                      _ptr(topk_w_out, torch.float32, "topk_w_out"), w, n,
                                      _stream(stream))
    _check("moe_forward_shared", rc)


# ---------------------------------------------------------------------------------------
# FP8 (e4m3) experts: codes are torch.uint8 tensors, scales torch.float32
# ---------------------------------------------------------------------------------------

def moe_workspace_size_fp8(p: Problem) -> int:
    """Workspace bytes for moe_forward_fp8 (0: invalid or unsupported on the FP8 path)."""
    return int(library().moe_workspace_size_fp8(ctypes.byref(p)))


def moe_quantize_experts_fp8(p, W1, W2, W1q, s1, W2q, s2, stream=None):
    """W1 [E, H, w1_cols], W2 [E, F, H] bf16 -> W1q [E, w1_cols, H], W2q [E, H, F] uint8 codes
    and per-column scales s1 [E, w1_cols], s2 [E, H] float32."""
    bf, u8, f32 = torch.bfloat16, torch.uint8, torch.float32
    rc = library().moe_quantize_experts_fp8(ctypes.byref(p), _ptr(W1, bf, "W1"), _ptr(W2, bf, "W2"),
                                            _ptr(W1q, u8, "W1q"), _ptr(s1, f32, "s1"),
                                            _ptr(W2q, u8, "W2q"), _ptr(s2, f32, "s2"),
                                            _stream(stream))
    _check("moe_quantize_experts_fp8", rc)


def moe_quantize_rows_fp8(src, dst, scale, stream=None):
    """src [rows, cols] bf16 -> dst [rows, cols] uint8 codes, scale [rows] float32."""
    rows, cols = src.shape
    rc = library().moe_quantize_rows_fp8(_ptr(src, torch.bfloat16, "src"), ctypes.c_int64(rows),
                                         cols, _ptr(dst, torch.uint8, "dst"),
                                         _ptr(scale, torch.float32, "scale"), _stream(stream))
    _check("moe_quantize_rows_fp8", rc)


def _fp8_args(p, x, Wg, bias, W1q, s1, W2q, s2, out, topk_idx_out, topk_w_out):
    bf, u8, f32 = torch.bfloat16, torch.uint8, torch.float32
    return (ctypes.byref(p), _ptr(x, bf, "x"), _ptr(Wg, bf, "Wg"), _ptr(bias, f32, "bias"),
            _ptr(W1q, u8, "W1q"), _ptr(s1, f32, "s1"), _ptr(W2q, u8, "W2q"), _ptr(s2, f32, "s2"),
            _ptr(out, bf, "out"), _ptr(topk_idx_out, torch.int32, "topk_idx_out"),
            _ptr(topk_w_out, f32, "topk_w_out"))


def moe_forward_fp8(p, x, Wg, bias, W1q, s1, W2q, s2, out, ws, topk_idx_out=None,
                    topk_w_out=None, stream=None):
    """The layer with e4m3 experts (codes and scales from moe_quantize_experts_fp8)."""
    w, n = _ws(ws)
    rc = library().moe_forward_fp8(*_fp8_args(p, x, Wg, bias, W1q, s1, W2q, s2, out, topk_idx_out,
                                              topk_w_out), w, n, _stream(stream))
    _check("moe_forward_fp8", rc)


def moe_forward_fp8_staged(p, x, Wg, bias, W1q, s1, W2q, s2, out, ws, events, topk_idx_out=None,
                           topk_w_out=None, stream=None):
    """moe_forward_fp8 with MOE_NUM_STAGE_EVENTS timing events at the stage boundaries."""
    w, n = _ws(ws)
    if len(events) != MOE_NUM_STAGE_EVENTS:
        raise ValueError(f"need {MOE_NUM_STAGE_EVENTS} events")
    for ev in events:
        if ev.cuda_event == 0:
            ev.record()
    arr = (ctypes.c_void_p * MOE_NUM_STAGE_EVENTS)(*[ctypes.c_void_p(e.cuda_event) for e in events])
    rc = library().moe_forward_fp8_staged(*_fp8_args(p, x, Wg, bias, W1q, s1, W2q, s2, out,
                                                     topk_idx_out, topk_w_out), w, n,
                                          _stream(stream), arr, MOE_NUM_STAGE_EVENTS)
    _check("moe_forward_fp8_staged", rc)


def moe_experts_forward(p, x, expert, gate, W1, W2, out, ws, stream=None):
    """out[r] = gate[r] * FFN_{expert[r]}(x[r]) for rows with known routing (p.top_k == 1)."""
    bf = torch.bfloat16
    w, n = _ws(ws)
    rc = library().moe_experts_forward(ctypes.byref(p), _ptr(x, bf, "x"),
                                       _ptr(expert, torch.int32, "expert"),
                                       _ptr(gate, torch.float32, "gate"), _ptr(W1, bf, "W1"),
                                       _ptr(W2, bf, "W2"), _ptr(out, bf, "out"), w, n,
                                       _stream(stream))
    _check("moe_experts_forward", rc)


def moe_experts_forward_n(p, x, expert, gate, n_rows, W1, W2, out, ws, stream=None):
    """moe_experts_forward on the first n_rows[0] rows (n_rows: a CUDA int32 tensor read on
    the device); rows past it are not computed and their output rows are left untouched."""
    bf = torch.bfloat16
    w, n = _ws(ws)
    rc = library().moe_experts_forward_n(ctypes.byref(p), _ptr(x, bf, "x"),
                                         _ptr(expert, torch.int32, "expert"),
                                         _ptr(gate, torch.float32, "gate"),
                                         _ptr(n_rows, torch.int32, "n_rows"), _ptr(W1, bf, "W1"),
                                         _ptr(W2, bf, "W2"), _ptr(out, bf, "out"), w, n,
                                         _stream(stream))
    _check("moe_experts_forward_n", rc)


def moe_ep_publish_counts(p, world, rank, offsets, tables, stream=None):
    """Row `rank` of every rank's counts table (tables: CUDA int64 tensor of world device
    addresses) = this rank's rows per destination, from the dispatch's [E+1] offsets."""
    rc = library().moe_ep_publish_counts(ctypes.byref(p), int(world), int(rank),
                                         _ptr(offsets, torch.int32, "offsets"),
                                         _ptr(tables, torch.int64, "tables"), _stream(stream))
    _check("moe_ep_publish_counts", rc)


def moe_ep_scatter(p, world, rank, x, topk_idx, topk_w, offsets, padded_offsets, inv_pos, table,
                   rows, ids, gates, origin, recv_cap, n_recv, ws, stream=None):
    """Stores every routed pair of this rank into its destination's receive buffers (the
    address arguments rows / ids / gates / origin: CUDA int64 tensors of world device
    addresses); n_recv[0] = rows this rank receives."""
    i64 = torch.int64
    w, n = _ws(ws)
    rc = library().moe_ep_scatter(
        ctypes.byref(p), int(world), int(rank), _ptr(x, torch.bfloat16, "x"),
        _ptr(topk_idx, torch.int32, "topk_idx"), _ptr(topk_w, torch.float32, "topk_w"),
        _ptr(offsets, torch.int32, "offsets"), _ptr(padded_offsets, torch.int32, "padded_offsets"),
        _ptr(inv_pos, torch.int32, "inv_pos"), _ptr(table, torch.int32, "table"),
        _ptr(rows, i64, "rows"), _ptr(ids, i64, "ids"), _ptr(gates, i64, "gates"),
        _ptr(origin, i64, "origin"), int(recv_cap), _ptr(n_recv, torch.int32, "n_recv"), w, n,
        _stream(stream))
    _check("moe_ep_scatter", rc)


def moe_ep_return(H, world, y, origin, n_recv, recv_cap, back, back_rows, ws, stream=None):
    """Stores each received row's expert output into its origin rank's return buffer (back:
    CUDA int64 tensor of world device addresses)."""
    rc = library().moe_ep_return(int(H), int(world), _ptr(y, torch.bfloat16, "y"),
                                 _ptr(origin, torch.int64, "origin"),
                                 _ptr(n_recv, torch.int32, "n_recv"), int(recv_cap),
                                 _ptr(back, torch.int64, "back"), int(back_rows),
                                 _ptr(ws, torch.uint8, "ws"), _stream(stream))
    _check("moe_ep_return", rc)


def moe_backward_workspace_size(p: Problem) -> int:
    """Workspace bytes for moe_backward (0: invalid or unsupported shape / gate mode)."""
    return int(library().moe_backward_workspace_size(ctypes.byref(p)))


def moe_backward(p, x, Wg, bias, W1, W2, dout, dx, dWg, dbias, dW1, dW2, ws, stream=None):
    """Gradients of the layer: dx, dW1, dW2 bf16; dWg [H, E], dbias [E] float32."""
    bf, f32 = torch.bfloat16, torch.float32
    w, n = _ws(ws)
    rc = library().moe_backward(ctypes.byref(p), _ptr(x, bf, "x"), _ptr(Wg, bf, "Wg"),
                                _ptr(bias, f32, "bias"), _ptr(W1, bf, "W1"), _ptr(W2, bf, "W2"),
                                _ptr(dout, bf, "dout"), _ptr(dx, bf, "dx"), _ptr(dWg, f32, "dWg"),
                                _ptr(dbias, f32, "dbias"), _ptr(dW1, bf, "dW1"),
                                _ptr(dW2, bf, "dW2"), w, n, _stream(stream))
    _check("moe_backward", rc)


def moe_combine(p, ys, inv_pos, out, ws=None, stream=None):
    bf = torch.bfloat16
    if ws is None:
        w, n = None, ctypes.c_size_t(0)
    else:
        w, n = _ws(ws)
    rc = library().moe_combine(ctypes.byref(p), _ptr(ys, bf, "ys"), ctypes.c_int64(ys.shape[0]),
                               _ptr(inv_pos, torch.int32, "inv_pos"), _ptr(out, bf, "out"), w, n,
                               _stream(stream))
    _check("moe_combine", rc)


def moe_get_device_status(ws, stream=None) -> int:
    """Synchronise the stream, read and clear the device status word; returns the code."""
    return int(library().moe_get_device_status(_ptr(ws, torch.uint8, "ws"), _stream(stream)))


def moe_set_wait_timeout_ns(ns: int) -> int:
    return int(library().moe_set_wait_timeout_ns(int(ns)))


GEMM_AUTO, GEMM_SINGLE_CTA, GEMM_CTA_PAIR, GEMM_FUSED, GEMM_FUSED_LAYERS = 0, 1, 2, 3, 4
ROUTER_AUTO, ROUTER_SEQUENTIAL, ROUTER_FILTER = 0, 1, 2
ORDER_EXPERT, ORDER_MIXED, ORDER_NARROW, ORDER_PHASED = 0, 1, 2, 3


def moe_set_fault_injection(layer0_item: int) -> int:
    """Test hook: withhold the ready signal of one layer0 work item of the fused kernel."""
    return int(library().moe_set_fault_injection(int(layer0_item)))


def moe_set_schedule_trace(records, capacity: int) -> None:
    """Record the persistent launch's schedule into ``records`` (a CUDA uint64/int64 tensor of
    at least 4 + 4 * capacity elements; element 0 counts the records), or switch the trace off
    with ``records=None``."""
    if records is None:
        rc = int(library().moe_set_schedule_trace(None, 0))
    else:
        if records.numel() < 4 + 4 * int(capacity) or records.element_size() != 8:
            raise ValueError("records: need 4 + 4 * capacity 64-bit elements")
        rc = int(library().moe_set_schedule_trace(ctypes.c_void_p(records.data_ptr()),
                                                 int(capacity)))
    if rc != 0:
        raise MoeError("moe_set_schedule_trace", rc)


def moe_set_work_order(order: int) -> int:
    """ORDER_EXPERT, ORDER_MIXED, ORDER_NARROW or ORDER_PHASED: how the single-CTA grouped
    GEMMs treat experts with a single m-tile. Returns the previous order."""
    rc = int(library().moe_set_work_order(int(order)))
    if rc < 0:
        raise ValueError(f"unknown work order {order}")
    return rc


def moe_set_router_mode(mode: int) -> int:
    """Select the router variant for many experts (ROUTER_AUTO, ROUTER_SEQUENTIAL or
    ROUTER_FILTER); returns the previous mode. All give the same routing and gates."""
    rc = int(library().moe_set_router_mode(int(mode)))
    if rc < 0:
        raise ValueError(f"unknown router mode {mode}")
    return rc


def moe_set_gemm_mode(mode: int) -> int:
    """Select the grouped-GEMM variant of later launches; returns the previous mode."""
    rc = int(library().moe_set_gemm_mode(int(mode)))
    if rc < 0:
        raise ValueError(f"unknown GEMM mode {mode}")
    return rc


def moe_set_whole_layer_launch(on: bool) -> bool:
    """Routing and dispatch inside the persistent launch where it applies (on by default);
    returns the previous setting."""
    return bool(library().moe_set_whole_layer_launch(1 if on else 0))


def moe_ep_buffer_sizes(p: Problem, world: int) -> list[int]:
    """Bytes of each of a rank's exchange buffers (EP_BUFFERS order)."""
    sizes = (ctypes.c_int64 * len(EP_BUFFERS))()
    rc = library().moe_ep_buffer_sizes(ctypes.byref(p), int(world), sizes)
    _check("moe_ep_buffer_sizes", rc)
    return [int(v) for v in sizes]


def moe_ep_workspace_size(p: Problem, world: int) -> int:
    n = int(library().moe_ep_workspace_size(ctypes.byref(p), int(world)))
    if n == 0:
        raise MoeError("moe_ep_workspace_size", -1)
    return n


def ep_rank(p: Problem, world: int, rank: int, epoch: int, x, Wg, bias, W1, W2, out, ws,
            buffers, topk_idx=None, topk_w=None) -> EpRank:
    """The moe_ep_rank of one rank. buffers[b][d]: rank d's buffer b as an int (its address on
    this GPU) or a tensor on this GPU."""
    r = EpRank()
    r.p = p
    r.world, r.rank, r.epoch = int(world), int(rank), int(epoch)
    r.x = _ptr(x, torch.bfloat16, "x")
    r.Wg = _ptr(Wg, torch.bfloat16, "Wg")
    r.bias = _ptr(bias, torch.float32, "bias")
    r.W1 = _ptr(W1, torch.bfloat16, "W1")
    r.W2 = _ptr(W2, torch.bfloat16, "W2")
    r.out = _ptr(out, torch.bfloat16, "out")
    r.topk_idx = _ptr(topk_idx, torch.int32, "topk_idx")
    r.topk_w = _ptr(topk_w, torch.float32, "topk_w")
    r.ws = _ptr(ws, torch.uint8, "ws")
    r.ws_bytes = ws.numel()
    for b in range(len(EP_BUFFERS)):
        for d in range(world):
            v = buffers[b][d]
            r.buf[b][d] = v if isinstance(v, int) else v.data_ptr()
    return r


def moe_ep_layer_forward(ranks, stream=None):
    """One launch for the ranks in `ranks` (EpRank structures; all on this GPU)."""
    n = len(ranks)
    arr = (EpRank * n)(*ranks)
    rc = library().moe_ep_layer_forward(arr, n, _stream(stream))
    _check("moe_ep_layer_forward", rc)
