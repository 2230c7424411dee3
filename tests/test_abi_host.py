"""Host-side checks of the C ABI that need no GPU.

The library must load and export every function ``include/*.h`` declares; argument errors must be reported before any device work; a host
without a usable device must get MOE_ERR_DEVICE rather than a crash.
"""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def mx():
    from tests.helpers import build_library
    build_library()
    import mxfp4_moe_expert_router_b200 as m
    return m


def _declared():
    names = set()
    for f in os.listdir(os.path.join(ROOT, "include")):
        if f.endswith(".h"):
            src = open(os.path.join(ROOT, "include", f)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names |= set(re.findall(r"^\s*(?:MOE_API\s+)?(?:int32_t|int64_t|void|const char\*)\s+(\w+)\s*\(", src, re.M))
    return names


def test_header_declares_the_boundary():
    assert {"mxfp4_quantize", "moe_mxfp4_create", "moe_route", "moe_forward",
            "moe_status", "moe_mxfp4_destroy"} <= _declared()


def test_library_exports_every_declared_symbol(mx):
    lib = ctypes.CDLL(mx.LIB_PATH)
    for name in _declared():
        assert hasattr(lib, name), name
    assert set(mx.EXPORTS) == _declared()


def test_exported_dynamic_symbols_are_only_the_abi(mx):
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", mx.LIB_PATH], capture_output=True, text=True).stdout
    exported = {ln.split()[-1] for ln in out.splitlines() if " T " in ln}
    ours = {s for s in exported if s.startswith(("moe_", "mxfp4_", "spec_"))}
    assert ours == _declared()


def test_status_strings(mx):
    assert mx.status_str(0) == "ok"
    assert mx.status_str(mx.MOE_ERR_TIMEOUT) == "device-side wait timed out"
    assert mx.status_str(99) == "unknown status"


def test_quantize_argument_errors(mx):
    q = mx.lib.mxfp4_quantize
    p = ctypes.c_void_p(1 << 20)
    assert q(p, 4, 31, p, p, None) == mx.MOE_ERR_INVALID_ARG
    assert q(p, 4, 0, p, p, None) == mx.MOE_ERR_INVALID_ARG
    assert q(p, -1, 32, p, p, None) == mx.MOE_ERR_INVALID_ARG
    assert q(None, 4, 32, p, p, None) == mx.MOE_ERR_INVALID_ARG
    assert q(ctypes.c_void_p((1 << 20) + 8), 4, 32, p, p, None) == mx.MOE_ERR_INVALID_ARG
    assert q(None, 0, 32, None, None, None) == mx.MOE_OK  # empty input is a no-op


def _create(mx, cfg, ptr=1 << 20, bias=False):
    arr = (ctypes.c_void_p * cfg.num_layers)(*([ptr] * cfg.num_layers))
    pp = ctypes.cast(arr, ctypes.POINTER(ctypes.c_void_p))
    h = ctypes.c_void_p(0)
    st = mx.lib.moe_mxfp4_create(ctypes.byref(cfg), pp, pp, pp, pp, pp, pp, pp,
                                 pp if bias else None, None, ctypes.byref(h))
    return st, h


@pytest.mark.parametrize("fields,status", [
    ((256, 128, 8, 2, 9, 1, 1e-6), None),
    ((0, 128, 8, 2, 9, 1, 1e-6), 1), ((256, 128, 8, 9, 9, 1, 1e-6), 1),
    ((256, 128, 8, 2, 0, 1, 1e-6), 1), ((256, 128, 8, 2, 9, 0, 1e-6), 1),
    ((256, 128, 8, 2, 9, 1, -1.0), 1),
    ((250, 128, 8, 2, 9, 1, 1e-6), 2), ((256, 100, 8, 2, 9, 1, 1e-6), 2),
    ((16384, 128, 8, 2, 9, 1, 1e-6), 2), ((256, 128, 1024, 2, 9, 1, 1e-6), 2),
    ((256, 128, 64, 33, 9, 1, 1e-6), 2), ((256, 128, 8, 2, 9, 17, 1e-6), 2),
])
def test_create_validation(mx, fields, status):
    cfg = mx.MoeConfig(*fields)
    st, h = _create(mx, cfg)
    if status is None:  # valid config: no device here, or invalid fake pointers on a GPU machine
        import torch
        assert st == (mx.MOE_ERR_DEVICE if not torch.cuda.is_available() else st)
    else:
        assert st == status
    assert not h.value


def test_create_rejects_null_and_misaligned(mx):
    cfg = mx.MoeConfig(256, 128, 8, 2, 9, 2, 1e-6)
    assert _create(mx, cfg, ptr=0)[0] == mx.MOE_ERR_INVALID_ARG
    assert _create(mx, cfg, ptr=(1 << 20) + 4)[0] == mx.MOE_ERR_INVALID_ARG
    h = ctypes.c_void_p(0)
    assert mx.lib.moe_mxfp4_create(None, None, None, None, None, None, None, None, None, None,
                                   ctypes.byref(h)) == mx.MOE_ERR_INVALID_ARG


def test_null_handle_calls(mx):
    p = ctypes.c_void_p(1 << 20)
    assert mx.lib.moe_forward(None, p, 9, p, None, None) == mx.MOE_ERR_INVALID_ARG
    assert mx.lib.moe_route(None, 0, p, 9, p, p, p, p, p, p, None) == mx.MOE_ERR_INVALID_ARG
    assert mx.lib.moe_forward_host(None, p, 9, p, None) == mx.MOE_ERR_INVALID_ARG
    assert mx.lib.moe_status(None, None) == mx.MOE_ERR_INVALID_ARG
    assert mx.lib.moe_set_timeout_ns(None, 5) == mx.MOE_ERR_INVALID_ARG
    assert mx.lib.moe_engine_grid(None) == 0
    mx.lib.moe_mxfp4_destroy(None)  # no-op
    assert mx.lib.moe_forward_ops(None, p, 9, p, None, 0, None) == mx.MOE_ERR_INVALID_ARG


def test_spec_verify_workspace_bounds(mx):
    ws = mx.lib.spec_verify_workspace_bytes
    assert ws(1, 8, 152064) > 0
    assert ws(64, 8, 152064) > ws(1, 8, 152064)
    assert ws(1, 0, 10) > 0
    for bad in [(0, 8, 100), (1, -1, 100), (1, 17, 100), (1, 8, 0), (1, 8, (1 << 22) + 1)]:
        assert ws(*bad) == -1, bad


def test_spec_verify_argument_errors(mx):
    f = mx.lib.spec_verify
    p = ctypes.c_void_p(1 << 20)
    n = mx.lib.spec_verify_workspace_bytes(2, 8, 1000)
    assert f(p, p, p, p, p, 0, 8, 1000, p, p, p, n, None) == mx.MOE_OK  # no blocks: no-op
    assert f(p, p, p, p, p, -1, 8, 1000, p, p, p, n, None) == mx.MOE_ERR_INVALID_ARG
    assert f(p, p, p, p, p, 2, 8, 1000, p, p, p, n - 8, None) == mx.MOE_ERR_INVALID_ARG  # workspace too small
    assert f(None, p, p, p, p, 2, 8, 1000, p, p, p, n, None) == mx.MOE_ERR_INVALID_ARG
    assert f(p, None, p, p, p, 2, 8, 1000, p, p, p, n, None) == mx.MOE_ERR_INVALID_ARG
    assert f(p, p, p, ctypes.c_void_p((1 << 20) + 4), p, 2, 8, 1000, p, p, p, n, None) == mx.MOE_ERR_INVALID_ARG
    assert f(p, p, p, p, p, 2, 8, 1000, p, p, ctypes.c_void_p((1 << 20) + 8), n, None) == mx.MOE_ERR_INVALID_ARG
    assert f(p, p, p, p, p, 2, 17, 1000, p, p, p, n, None) == mx.MOE_ERR_INVALID_ARG
    assert mx.lib.spec_verify_status(None, None) == mx.MOE_ERR_INVALID_ARG
    import torch
    if not torch.cuda.is_available():  # valid arguments, no device
        assert f(p, p, p, p, p, 2, 8, 1000, p, p, p, n, None) == mx.MOE_ERR_DEVICE
        # G == 0 needs no draft arrays
        n0 = mx.lib.spec_verify_workspace_bytes(2, 0, 1000)
        assert f(p, None, None, None, p, 2, 0, 1000, p, p, p, n0, None) == mx.MOE_ERR_DEVICE


def test_partial_and_round_argument_errors(mx):
    p = ctypes.c_void_p(1 << 20)
    assert mx.lib.moe_forward_partial(None, p, 9, p, None) == mx.MOE_ERR_INVALID_ARG
    assert mx.lib.moe_round_bf16(p, p, -1, None) == mx.MOE_ERR_INVALID_ARG
    assert mx.lib.moe_round_bf16(None, p, 4, None) == mx.MOE_ERR_INVALID_ARG
    assert mx.lib.moe_round_bf16(ctypes.c_void_p((1 << 20) + 2), p, 4, None) == mx.MOE_ERR_INVALID_ARG
    assert mx.lib.moe_round_bf16(None, None, 0, None) == mx.MOE_OK


def test_route_static_size_formula_on_the_host(mx):
    """The header's working-memory formula of moe_route_static: the first T beyond it is
    refused before any device work (so this runs without a GPU)."""
    p = ctypes.c_void_p(1 << 20)
    limit = mx.MOE_ROUTE_STATIC_SCRATCH_BYTES
    for H, E, k in [(256, 16, 4), (4096, 128, 8), (7168, 256, 8)]:
        T = 1
        while 64 * T * E + 36 * min(E, T * k) + 17 * T * k <= limit:
            T += 1
        assert mx.lib.moe_route_static(p, T, H, p, None, E, k, p, p, p, p, p, p, None) == \
            mx.MOE_ERR_UNSUPPORTED_SHAPE, (H, E, k, T)
    import torch
    if not torch.cuda.is_available():  # no device: the status query has nothing to report
        assert mx.lib.moe_route_static_status(None) in (mx.MOE_OK, mx.MOE_ERR_DEVICE, mx.MOE_ERR_CUDA)
