"""Host-side checks of the C ABI (no GPU needed).

The library must load, export every function include/moelora.h declares, and
reject bad arguments on the host before any CUDA call (so these run on a
CPU-only machine).  Workspace sizing is checked against its own formula.
"""
import ctypes
import os
import re

import pytest

import mixture_experts_lora_b200 as ml

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moelora.h")


@pytest.fixture(scope="module")
def L():
    from mixture_experts_lora_b200 import build
    build.build(quiet=True)
    return ml.lib()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z_0-9]+)\s*\(", src)))


def test_header_declares_the_abi():
    names = declared_functions()
    assert set(ml.EXPORTED) == set(names)


def test_library_exports_every_declared_symbol(L):
    for name in declared_functions():
        assert hasattr(L, name), name
    nm = os.popen(f"nm -D --defined-only {ml.LIB_PATH}").read()
    for name in declared_functions():
        assert re.search(rf"\bT {name}\b", nm), name


def test_status_strings(L):
    for s in range(8):
        assert ml.status_string(s)
    assert ml.status_string(ml.MOE_ERR_WORKSPACE) == "workspace too small"


def dims(**kw):
    base = dict(T=256, m=128, n=64, E=8, k=2, r=8, scale=2.0)
    base.update(kw)
    return ml.make_dims(**base)


def test_workspace_bytes_supported_and_not(L):
    assert ml.moe_workspace_bytes(dims()) > 0
    for bad in (dict(k=0), dict(k=33, E=64), dict(E=1025), dict(m=120), dict(n=8), dict(r=12),
                dict(r=136), dict(r=44), dict(E=1, k=2), dict(T=-1)):
        assert ml.moe_workspace_bytes(dims(**bad)) == 0, bad


def test_workspace_grows_with_tokens(L):
    a = ml.moe_workspace_bytes(dims(T=256))
    b = ml.moe_workspace_bytes(dims(T=4096))
    P = 4096 * 2
    assert b > a
    # holds at least the sorted rows, dGU and the two rank-r buffers
    assert b >= P * 128 * 2 + P * 128 * 2 + 2 * P * 16 * 2


def test_host_validation_returns_before_launch(L):
    P = ctypes.c_void_p
    null = None
    # route: unsupported k, negative T
    assert L.moe_route_topk(null, 4, 8, 0, null, null, null) == ml.MOE_ERR_UNSUPPORTED
    assert L.moe_route_topk(null, 4, 8, 9, null, null, null) == ml.MOE_ERR_UNSUPPORTED
    assert L.moe_route_topk(null, -1, 8, 2, null, null, null) == ml.MOE_ERR_INVALID_ARG
    assert L.moe_route_topk(null, 4, 8, 2, null, null, null) == ml.MOE_ERR_INVALID_ARG
    assert L.moe_route_topk(null, 0, 8, 2, null, null, null) == ml.MOE_OK  # empty input
    # permute: NULL workspace, then too small a workspace
    fake = P(256)
    assert L.moe_permute(fake, 4, 2, 8, fake, fake, fake, fake, null, 0, null) == ml.MOE_ERR_INVALID_ARG
    assert L.moe_permute(fake, 4, 2, 8, fake, fake, fake, fake, fake, 8, null) == ml.MOE_ERR_WORKSPACE
    # forward: bad dims, NULL / misaligned pointers, small workspace
    d = dims()
    ptrs = [P(4096)] * 16
    assert L.moe_grouped_gemm_lora_fwd(ctypes.byref(dims(m=100)), *ptrs, 1 << 30, null) == ml.MOE_ERR_UNSUPPORTED
    assert L.moe_grouped_gemm_lora_fwd(None, *ptrs, 1 << 30, null) == ml.MOE_ERR_INVALID_ARG
    bad = list(ptrs)
    bad[0] = P(4098)
    assert L.moe_grouped_gemm_lora_fwd(ctypes.byref(d), *bad, 1 << 30, null) == ml.MOE_ERR_INVALID_ARG
    bad[0] = None
    assert L.moe_grouped_gemm_lora_fwd(ctypes.byref(d), *bad, 1 << 30, null) == ml.MOE_ERR_INVALID_ARG
    assert L.moe_grouped_gemm_lora_fwd(ctypes.byref(d), *ptrs, 16, null) == ml.MOE_ERR_WORKSPACE
    nan = ml.make_dims(256, 128, 64, 8, 2, 8, float("nan"))
    assert L.moe_grouped_gemm_lora_fwd(ctypes.byref(nan), *ptrs, 1 << 30, null) == ml.MOE_ERR_INVALID_ARG
    # empty forward is a no-op
    assert L.moe_grouped_gemm_lora_fwd(ctypes.byref(dims(T=0)), *ptrs, 0, null) == ml.MOE_OK
    # backward: misaligned gradient output, small workspace
    bptrs = [P(4096)] * 21
    bb = list(bptrs)
    bb[16] = P(4100)
    assert L.moe_grouped_gemm_lora_bwd(ctypes.byref(d), *bb, 1 << 30, null) == ml.MOE_ERR_INVALID_ARG
    assert L.moe_grouped_gemm_lora_bwd(ctypes.byref(d), *bptrs, 16, null) == ml.MOE_ERR_WORKSPACE
    # combine
    assert L.moe_unpermute_combine(fake, null, fake, 4, 2, 12, fake, null) == ml.MOE_ERR_UNSUPPORTED
    assert L.moe_unpermute_combine(fake, null, fake, -1, 2, 16, fake, null) == ml.MOE_ERR_INVALID_ARG
    assert L.moe_unpermute_combine(fake, null, fake, 0, 2, 16, fake, null) == ml.MOE_OK


def test_full_backward_host_validation(L):
    P = ctypes.c_void_p
    d = dims()
    ptrs = [P(4096)] * 23         # ... dX_sorted, dW_gu (16), dW_d (17), dA_gu .. dB_d (18-21), ws

    def call(p, ws_bytes=1 << 30):
        return L.moe_grouped_gemm_full_bwd(ctypes.byref(d), *p, ws_bytes, None)
    bad = list(ptrs)
    bad[16] = None                # the expert-weight gradients are required
    assert call(bad) == ml.MOE_ERR_INVALID_ARG
    bad = list(ptrs)
    bad[19] = None                # adapter gradients: all four or none
    assert call(bad) == ml.MOE_ERR_INVALID_ARG
    bad = list(ptrs)
    bad[17] = P(4100)             # misaligned dW_d
    assert call(bad) == ml.MOE_ERR_INVALID_ARG
    assert call(ptrs, 16) == ml.MOE_ERR_WORKSPACE
    no_adapters = list(ptrs)
    no_adapters[18:22] = [None] * 4
    assert call(no_adapters, 16) == ml.MOE_ERR_WORKSPACE
    assert L.moe_grouped_gemm_full_bwd(ctypes.byref(dims(m=100)), *ptrs, 1 << 30, None) == ml.MOE_ERR_UNSUPPORTED
    # the LoRA backward keeps requiring its adapter gradients
    lb = [P(4096)] * 21
    lb[18] = None
    assert L.moe_grouped_gemm_lora_bwd(ctypes.byref(d), *lb, 1 << 30, None) == ml.MOE_ERR_INVALID_ARG


def test_check_permutation_host_validation(L):
    fake = ctypes.c_void_p(256)
    null = None
    assert L.moe_check_permutation(fake, 4, 0, 8, fake, fake, fake, fake, null) == ml.MOE_ERR_UNSUPPORTED
    assert L.moe_check_permutation(fake, -1, 2, 8, fake, fake, fake, fake, null) == ml.MOE_ERR_INVALID_ARG
    assert L.moe_check_permutation(fake, 4, 2, 8, null, fake, fake, fake, null) == ml.MOE_ERR_INVALID_ARG
    assert L.moe_check_permutation(null, 4, 2, 8, fake, fake, fake, fake, null) == ml.MOE_ERR_INVALID_ARG


def test_debug_checks_follow_the_environment(monkeypatch):
    monkeypatch.delenv("MOE_CHECK", raising=False)
    assert not ml.debug_checks()
    monkeypatch.setenv("MOE_CHECK", "0")
    assert not ml.debug_checks()
    monkeypatch.setenv("MOE_CHECK", "1")
    assert ml.debug_checks()


def test_router_backward_host_validation(L):
    null = None
    fake = ctypes.c_void_p(256)       # 16-byte aligned, never dereferenced
    odd = ctypes.c_void_p(258)
    args = lambda **kw: [kw.get("dY", fake), kw.get("ys", fake), fake, fake, fake, kw.get("T", 4),
                         kw.get("k", 2), kw.get("E", 8), kw.get("m", 64), kw.get("out", fake), null]
    assert L.moe_router_backward(*args(k=0)) == ml.MOE_ERR_UNSUPPORTED
    assert L.moe_router_backward(*args(k=33, E=64)) == ml.MOE_ERR_UNSUPPORTED
    assert L.moe_router_backward(*args(E=1)) == ml.MOE_ERR_UNSUPPORTED
    assert L.moe_router_backward(*args(m=12)) == ml.MOE_ERR_UNSUPPORTED
    assert L.moe_router_backward(*args(m=4)) == ml.MOE_ERR_INVALID_ARG
    assert L.moe_router_backward(*args(T=-1)) == ml.MOE_ERR_INVALID_ARG
    assert L.moe_router_backward(*args(dY=odd)) == ml.MOE_ERR_INVALID_ARG
    assert L.moe_router_backward(*args(out=null)) == ml.MOE_ERR_INVALID_ARG
    assert L.moe_router_backward(*args(T=0, out=null)) == ml.MOE_OK   # empty input


def test_binding_raises_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(ml, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(ml, "_lib_handle", None)
    with pytest.raises(RuntimeError):
        ml.lib()


def test_selftest_bounded_wait_checks_its_arguments(L):
    # out-of-range limits and a NULL flag are refused on the host, before any launch
    assert L.moe_selftest_bounded_wait(999, ctypes.c_void_p(16), None) == ml.MOE_ERR_INVALID_ARG
    assert L.moe_selftest_bounded_wait(2_000_000_000, ctypes.c_void_p(16), None) == ml.MOE_ERR_INVALID_ARG
    assert L.moe_selftest_bounded_wait(1_000_000, None, None) == ml.MOE_ERR_INVALID_ARG


def test_route_permute_host_validation(L):
    P = ctypes.c_void_p
    fake, null = P(256), None
    args = lambda T, E, k, ws, wsb: (fake, T, E, k, fake, fake, fake, fake, fake, fake, ws, wsb, null)
    assert L.moe_route_permute(*args(4, 8, 0, fake, 1 << 20)) == ml.MOE_ERR_UNSUPPORTED
    assert L.moe_route_permute(*args(4, 8, 9, fake, 1 << 20)) == ml.MOE_ERR_UNSUPPORTED
    assert L.moe_route_permute(*args(-1, 8, 2, fake, 1 << 20)) == ml.MOE_ERR_INVALID_ARG
    assert L.moe_route_permute(*args(4, 8, 2, null, 0)) == ml.MOE_ERR_INVALID_ARG
    assert L.moe_route_permute(*args(4, 8, 2, fake, 8)) == ml.MOE_ERR_WORKSPACE
    # moe_workspace_bytes covers the routed histogram chunks for any k
    for k in (1, 3, 5, 8, 32):
        T, E = 1000, 64
        chunks = -(-T // (512 // k))
        assert ml.moe_workspace_bytes(dims(T=T, E=E, k=k)) >= (chunks * E + 32 * E + 1) * 4
