"""CPU checks of the C ABI library: it builds, loads, exports every function that
include/moe.h declares, and rejects bad arguments on the host (no kernel is launched and
no CUDA call is made on these paths)."""
import ctypes
import re
from pathlib import Path

import pytest

import mixture_experts_layer_forward_b200 as moe
from mixture_experts_layer_forward_b200 import build as native_build

ROOT = Path(__file__).resolve().parents[1]


@pytest.fixture(scope="module")
def lib():
    native_build.build_library()
    return moe.library()


def declared_functions():
    names = []
    for h in sorted((ROOT / "include").glob("*.h")):
        text = h.read_text()
        names += re.findall(r"^MOE_API\s+[^;(]*?\b(moe_\w+)\s*\(", text, flags=re.M)
    return names


def test_header_declares_the_entry_points():
    names = set(declared_functions())
    for n in ("moe_route", "moe_dispatch", "moe_forward", "moe_combine", "moe_workspace_size",
              "moe_get_device_status"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert names
    for n in names:
        assert hasattr(lib, n), f"{n} declared in include/ but not exported"


def test_only_declared_symbols_are_exported(lib):
    import subprocess

    out = subprocess.run(["nm", "-D", "--defined-only", str(moe.library_path())],
                         capture_output=True, text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    moe_syms = {s for s in exported if s.startswith("moe_")}
    assert moe_syms == set(declared_functions())


def test_host_side_argument_checks(lib):
    P = moe.Problem
    good = P.make(256, 256, 512, 8, 2)
    assert moe.moe_workspace_size(good) > 0
    assert moe.moe_padded_rows_max(good) == 256 * 2 + 8 * 127
    assert moe.moe_padded_rows_max(P.make(1, 256, 512, 8, 1)) == 1 + 1 * 127
    bad = [P.make(256, 256, 512, 8, 9),          # k > E
           P.make(-1, 256, 512, 8, 2),           # T < 0
           P.make(256, 0, 512, 8, 2),            # H = 0
           P.make(256, 256, 512, 8, 2, act=7),   # unknown activation
           P.make(256, 256, 512, 8, 2, gate=5)]  # unknown gate
    for p in bad:
        assert moe.moe_workspace_size(p) == 0
        assert lib.moe_forward(ctypes.byref(p), *([None] * 9), 0, None) == -1
    unsupported = [P.make(256, 100, 512, 8, 2),   # H % 64
                   P.make(256, 256, 96, 8, 2),    # F % 64
                   P.make(256, 256, 512, 2048, 2),  # E > 1024
                   P.make(256, 256, 512, 8, 2, m_tile=64)]
    for p in unsupported:
        assert moe.moe_workspace_size(p) == 0
        assert lib.moe_forward(ctypes.byref(p), *([None] * 9), 0, None) == -2
    # NULL pointers / short workspace are rejected before any CUDA call
    assert lib.moe_forward(ctypes.byref(good), *([None] * 9), 0, None) == -1
    fake = ctypes.c_void_p(1 << 20)
    args = [fake] * 6 + [None, None]
    assert lib.moe_forward(ctypes.byref(good), *args, fake, 16, None) == -3
    assert lib.moe_route(ctypes.byref(good), fake, fake, None, fake, fake, fake, 16, None) == -3
    # a gate matrix off the 16-byte boundary is rejected before any launch
    off = ctypes.c_void_p((1 << 20) + 2)
    assert lib.moe_route(ctypes.byref(good), fake, off, None, fake, fake, fake,
                         moe.moe_workspace_size(good), None) == -1
    assert lib.moe_route_noalloc(ctypes.byref(good), fake, off, None, fake, fake, None) == -1
    assert lib.moe_get_device_status(None, None) == -1
    assert lib.moe_set_schedule_trace(None, -1) == -1
    assert lib.moe_set_schedule_trace(None, 0) == 0
    assert lib.moe_status_string(-5) == b"MOE_ERR_DEVICE_TIMEOUT"


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    from mixture_experts_layer_forward_b200 import _native

    monkeypatch.setattr(_native, "LIB_PATH", tmp_path / "absent.so")
    monkeypatch.setattr(_native, "_lib", None)
    with pytest.raises(RuntimeError, match="no CPU fallback"):
        _native.library()


def test_forward_launch_count_follows_the_modes(lib):
    """moe_forward_launches: host logic only (router and GEMM choice), no GPU needed."""
    from mixture_experts_layer_forward_b200 import synth

    mixtral = moe.Problem.from_config(synth.CONFIGS["mixtral"])
    qwen2 = moe.Problem.from_config(synth.CONFIGS["qwen2"])
    decode = moe.Problem.from_config(synth.CONFIGS["skew_decode"])
    prev_r = moe.moe_set_router_mode(moe.ROUTER_AUTO)
    prev_g = moe.moe_set_gemm_mode(moe.GEMM_AUTO)
    prev_o = moe.moe_set_work_order(moe.ORDER_EXPERT)
    try:
        # router 1 (up to 32 experts, E % 8 == 0), 2 (more experts, sequential) or 3 (the
        # filter) + dispatch 3 (1 for T <= 256) + [x gather] + layer0, layer1, combine; the
        # bench layers gather x into sorted rows (T * k >= 128 E)
        # large batches (T*k >= 128 E) gather x into sorted rows and take the persistent
        # launch: router + dispatch 3 + gather + 1
        # (E <= 8: the persistent launch)
        # E = 8 with the one-launch router: the whole layer in the persistent launch
        assert moe.moe_forward_launches(mixtral) == 1
        assert moe.moe_set_whole_layer_launch(False) is True
        try:
            assert moe.moe_forward_launches(mixtral) == 6   # router, dispatch 3, gather, layers
        finally:
            moe.moe_set_whole_layer_launch(True)
        assert moe.moe_forward_launches(moe.Problem.make(1000, 256, 256, 8, 2)) == 1
        assert moe.moe_forward_launches(qwen2) == 10    # T*E >= 2^16: filter router
        assert moe.moe_forward_launches(decode) == 6    # T*E < 2^16: sequential, three layers
        phi35 = moe.Problem.from_config(synth.CONFIGS["phi35"])
        assert moe.moe_forward_launches(phi35) == 10    # E = 16: filter router
        moe.moe_set_router_mode(moe.ROUTER_FILTER)
        assert moe.moe_forward_launches(decode) == 7
        assert moe.moe_forward_launches(mixtral) == 8   # forced: E = 8 qualifies
        assert moe.moe_forward_launches(moe.Problem.make(64, 128, 128, 4, 2)) == 6  # E % 8
        moe.moe_set_router_mode(moe.ROUTER_SEQUENTIAL)
        assert moe.moe_forward_launches(mixtral) == 1   # the one-launch router again
        assert moe.moe_forward_launches(phi35) == 8     # E = 16: one-launch router
        assert moe.moe_forward_launches(moe.Problem.make(64, 128, 128, 4, 2)) == 6  # E % 8
        assert moe.moe_forward_launches(qwen2) == 9
        moe.moe_set_gemm_mode(moe.GEMM_FUSED)           # forced: the persistent launch
        assert moe.moe_forward_launches(qwen2) == 7
        moe.moe_set_gemm_mode(moe.GEMM_FUSED_LAYERS)    # layers in it, the combine after
        assert moe.moe_forward_launches(qwen2) == 8
        assert moe.moe_forward_launches(mixtral) == 7   # no whole-layer launch then
        moe.moe_set_gemm_mode(moe.GEMM_FUSED)
        moe.moe_set_gemm_mode(moe.GEMM_SINGLE_CTA)      # three layer launches
        assert moe.moe_forward_launches(qwen2) == 9
        moe.moe_set_work_order(moe.ORDER_NARROW)        # the same launches, SMs split inside
        assert moe.moe_forward_launches(qwen2) == 9
        moe.moe_set_gemm_mode(moe.GEMM_FUSED)           # forced on a decode batch: no gather
        assert moe.moe_forward_launches(decode) == 4
        moe.moe_set_gemm_mode(moe.GEMM_CTA_PAIR)        # gathers x; no narrow launches
        assert moe.moe_forward_launches(qwen2) == 9
        assert moe.moe_forward_launches(decode) == 7
        assert moe.moe_forward_launches(moe.Problem.make(0, 128, 128, 8, 2)) == 0
        moe.moe_set_gemm_mode(moe.GEMM_AUTO)
        assert moe.moe_forward_launches(moe.Problem.make(256, 128, 128, 8, 2)) == 5  # one chunk
        assert moe.moe_forward_launches(moe.Problem.make(257, 128, 128, 8, 2)) == 7  # two
        assert moe.moe_forward_launches(moe.Problem.make(4, 100, 128, 8, 2)) == -1  # H % 64
    finally:
        moe.moe_set_router_mode(prev_r)
        moe.moe_set_gemm_mode(prev_g)
        moe.moe_set_work_order(prev_o)
    with pytest.raises(ValueError):
        moe.moe_set_router_mode(7)
    with pytest.raises(ValueError):
        moe.moe_set_work_order(4)


def test_shared_expert_workspace_and_checks(lib):
    """Host-only checks of the shared-expert entry points (no kernel launched)."""
    p = moe.Problem.make(300, 256, 192, 16, 2)
    base = moe.moe_workspace_size(p)
    assert moe.moe_workspace_size_shared(p, 320) > base
    assert moe.moe_workspace_size_shared(p, 100) == 0      # F_s % 64
    assert moe.moe_workspace_size_shared(p, 0) == 0
    sh = moe.SharedExpert(320, None, None, None)            # no weights: invalid argument
    rc = lib.moe_forward_shared(ctypes.byref(p), None, None, None, None, None, ctypes.byref(sh),
                                None, None, None, None, 0, None)
    assert rc == -1


def test_route_uses_filter_follows_mode_and_shape(lib):
    skew = moe.Problem.make(4096, 7168, 2048, 256, 8)
    mixtral = moe.Problem.make(8192, 4096, 14336, 8, 2)
    assert moe.moe_route_uses_filter(skew) and not moe.moe_route_uses_filter(mixtral)
    prev = moe.moe_set_router_mode(moe.ROUTER_SEQUENTIAL)
    try:
        assert not moe.moe_route_uses_filter(skew)
        moe.moe_set_router_mode(moe.ROUTER_FILTER)
        assert moe.moe_route_uses_filter(mixtral)
    finally:
        moe.moe_set_router_mode(prev)


def test_fp8_workspace_and_argument_checks(lib):
    p = moe.Problem.make(300, 256, 256, 16, 2)
    assert moe.moe_workspace_size_fp8(p) > moe.moe_workspace_size(p)
    assert moe.moe_workspace_size_fp8(moe.Problem.make(300, 192, 256, 16, 2)) == 0  # H % 128
    assert moe.moe_workspace_size_fp8(moe.Problem.make(300, 256, 192, 16, 2)) == 0  # F % 128
    # host-detected errors: nothing is launched
    assert lib.moe_quantize_rows_fp8(None, 4, 12, None, None, None) == -1             # cols % 8
    assert lib.moe_quantize_experts_fp8(ctypes.byref(p), None, None, None, None, None, None,
                                        None) == -1
    assert lib.moe_forward_fp8(ctypes.byref(p), None, None, None, None, None, None, None, None,
                               None, None, None, 0, None) == -1


def test_backward_workspace_and_argument_checks(lib):
    p = moe.Problem.make(300, 256, 256, 16, 2)
    assert moe.moe_backward_workspace_size(p) > moe.moe_workspace_size(p)
    assert moe.moe_backward_workspace_size(moe.Problem.make(300, 256, 192, 16, 2)) == 0   # F % 128
    assert lib.moe_backward(ctypes.byref(p), *([None] * 12), 0, None) == -1


def _header_prototypes():
    text = "\n".join(h.read_text() for h in sorted((ROOT / "include").glob("*.h")))
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    protos = {}
    for m in re.finditer(r"MOE_API\s+([^;(]*?)\b(moe_\w+)\s*\(([^)]*)\)\s*;", text, flags=re.S):
        params = " ".join(m.group(3).split())
        plist = [] if params in ("", "void") else [q.strip() for q in params.split(",")]
        protos[m.group(2)] = (" ".join(m.group(1).split()), plist)
    return protos


def _ctype_kind(c_decl):
    """Category of a C parameter or return type: pointer, size, i64 or i32."""
    if "*" in c_decl:
        return "pointer"
    words = c_decl.replace("const ", "").split()
    base = words[0]
    if base == "size_t":
        return "size"
    if base == "int64_t":
        return "i64"
    if base in ("int", "int32_t", "moe_status"):
        return "i32"
    raise AssertionError(f"unexpected C type {c_decl!r}")


def _ctypes_kind(t):
    if t is ctypes.c_void_p or t is ctypes.c_char_p or (
            isinstance(t, type) and issubclass(t, ctypes._Pointer)):
        return "pointer"
    if t is ctypes.c_size_t:
        return "size"
    if t is ctypes.c_int64:
        return "i64"
    if t is ctypes.c_int:
        return "i32"
    raise AssertionError(f"unexpected ctypes type {t!r}")


def test_binding_signatures_match_the_header(lib):
    """Every prototype in include/ has a ctypes signature in the binding with the same number
    of arguments and the same kind (pointer, size_t, int64, int) of each argument and of the
    result: a parameter added on one side only would otherwise shift every later argument."""
    protos = _header_prototypes()
    assert set(protos) == set(declared_functions())
    for name, (ret, params) in protos.items():
        f = getattr(lib, name)
        assert f.argtypes is not None, f"{name}: no argtypes in the binding"
        assert len(f.argtypes) == len(params), (name, len(f.argtypes), len(params))
        for i, (c_decl, t) in enumerate(zip(params, f.argtypes)):
            assert _ctype_kind(c_decl) == _ctypes_kind(t), (name, i, c_decl, t)
        assert _ctype_kind(ret) == _ctypes_kind(f.restype), (name, ret, f.restype)


def test_every_entry_point_has_a_python_function():
    """The package exposes each C entry point under its own name (moe_status_string is used
    inside the binding's error messages)."""
    for name in declared_functions():
        if name != "moe_status_string":
            assert callable(getattr(moe, name, None)), name


def test_ep_layer_sizes_and_checks(lib):
    """Host-only: the exchange buffer sizes of the expert-parallel layer, and the shapes it
    refuses (no kernel launched)."""
    p = moe.Problem.make(8192, 4096, 14336, 8, 2)
    world = 2
    sizes = moe.moe_ep_buffer_sizes(p, world)
    recv_cap = world * 8192 * 2 + 4 * 127   # rows routed to E / world experts, each padded
    assert sizes == [world * 1024 * 8 * 4, world * 4, recv_cap * 4096 * 2, recv_cap * 4,
                     recv_cap * 8, (recv_cap // 128 + 1) * 4, 8192 * 2 * 4096 * 2, 8192 * 16 * 4]
    assert moe.moe_ep_workspace_size(p, world) > 0
    for bad_world in (0, 3, 9):            # must divide E = 8 and be at most 8
        assert lib.moe_ep_workspace_size(ctypes.byref(p), bad_world) == 0
    wide = moe.Problem.make(512, 256, 256, 64, 2)   # the one-launch router takes E <= 32
    assert lib.moe_ep_workspace_size(ctypes.byref(wide), 2) == 0
    assert lib.moe_ep_layer_forward(None, 1, None) == -1
    r = moe.EpRank()
    r.p = p
    r.world, r.rank, r.epoch = world, 0, 0          # epoch must be positive
    assert lib.moe_ep_layer_forward(ctypes.byref(r), 1, None) == -1
    assert lib.moe_ep_layer_forward(ctypes.byref(r), 5, None) == -1  # more ranks than one launch takes


@pytest.mark.parametrize("T,H,E,k,launches", [
    (512, 256, 8, 2, 1),     # T*k = 1024 = 128 E: sorted rows, the whole layer in one launch
    (511, 256, 8, 2, 7),     # T*k < 128 E: router, dispatch 3, layers 3 (rows gathered in-kernel)
    (256, 128, 8, 4, 1),     # k = 4: 1024 routed rows
    (1024, 128, 16, 2, 8),   # E = 16, T*E < 2^16: one-launch router, dispatch 3, gather, layers 3
    (20000, 256, 8, 2, 1),   # 128-token groups, more groups than SMs
    (600, 96, 8, 2, -1),     # H % 64 != 0: invalid
])
def test_whole_layer_plan_boundaries(lib, T, H, E, k, launches):
    """Host logic only: where the whole-layer launch applies (E = 8, T*k >= 128 E, the
    one-launch router) and what runs elsewhere."""
    prev = moe.moe_set_gemm_mode(moe.GEMM_AUTO)
    prev_r = moe.moe_set_router_mode(moe.ROUTER_AUTO)
    try:
        assert moe.moe_forward_launches(moe.Problem.make(T, H, 256, E, k)) == launches
    finally:
        moe.moe_set_gemm_mode(prev)
        moe.moe_set_router_mode(prev_r)


def test_ep_local_launch_refuses_too_many_ranks(lib):
    """Host-only: one launch carries at most EP_MAX_LOCAL ranks (checked before any launch),
    and the experts must split evenly over the ranks."""
    from mixture_experts_layer_forward_b200 import ep

    p = moe.Problem.make(64, 128, 128, 8, 2)
    n = moe.EP_MAX_LOCAL + 1
    with pytest.raises(ValueError):
        ep.ep_layer_forward_local(p, [None] * n, None, None, [None] * n, [None] * n, [None] * n,
                                  [None] * n, [None] * n, epoch=1)
    with pytest.raises(ValueError):
        ep.experts_per_rank(8, 3)
    assert ep.experts_per_rank(8, 4) == 2
