"""Host-only checks of the C ABI: the library loads, exports every function
include/w4a16.h declares, and rejects bad arguments before launching anything.

No test here reaches a kernel launch: every call fails validation first, so
the fake device addresses below are never dereferenced."""
import ctypes
import os
import re

import pytest

import w4a16_decode_gemv_b200 as w4
from w4a16_decode_gemv_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "w4a16.h")

OK, ERR_ARG, ERR_ALIGN, ERR_SHAPE, ERR_UNSUPPORTED, ERR_WORKSPACE = 0, -1, -2, -3, -4, -5
A = 0x10000          # a 16-byte aligned fake address (never dereferenced)
B = 0x20000
MIS = 0x10008        # 8-byte aligned only


@pytest.fixture(scope="module")
def lib():
    build.build()
    return w4.load_library()


def declared_functions():
    text = open(HEADER).read()
    return re.findall(r"W4A16_API\s+[\w\s\*]+?\b(\w+)\s*\(", text)


def test_header_declares_the_boundary():
    names = set(declared_functions())
    assert {"awq_act_scale", "awq_quantize_pack", "w4a16_gemm", "w4a16_gemm_workspace_size",
            "w4a16_gemm_check", "w4a16_last_error", "w4a16_layout_version"} <= names


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
        assert ctypes.cast(getattr(lib, name), ctypes.c_void_p).value


def test_layout_version(lib):
    assert lib.w4a16_layout_version() == 1


def _err(lib):
    return lib.w4a16_last_error().decode()


def test_quantize_pack_validation(lib):
    qp = lib.awq_quantize_pack
    assert qp(None, None, 8, 128, 128, 4, 0, A, A, A, None) == ERR_ARG
    assert "null" in _err(lib)
    assert qp(A, None, 0, 128, 128, 4, 0, A, A, A, None) == ERR_ARG
    assert qp(A, None, 8, 128, 128, 4, 7, A, A, A, None) == ERR_ARG
    assert qp(A, None, 8, 128, 64, 4, 0, A, A, A, None) == ERR_UNSUPPORTED
    assert qp(A, None, 8, 128, 128, 5, 0, A, A, A, None) == ERR_UNSUPPORTED
    assert qp(A, None, 8, 128, 128, 2, 1, A, A, A, None) == ERR_UNSUPPORTED
    assert qp(A, None, 8, 200, 128, 4, 0, A, A, A, None) == ERR_SHAPE
    assert qp(MIS, None, 8, 128, 128, 4, 0, A, A, A, None) == ERR_ALIGN
    assert qp(A, MIS, 8, 128, 128, 4, 0, A, A, A, None) == ERR_ALIGN
    assert qp(A, None, 8, 128, 128, 4, 0, A, A, MIS, None) == ERR_ALIGN
    assert qp(A, None, 1 << 20, 1 << 12, 128, 4, 0, A, A, A, None) == ERR_SHAPE


def test_act_scale_validation(lib):
    f = lib.awq_act_scale
    assert f(None, 4, 8, 0.5, A, None) == ERR_ARG
    assert f(A, 0, 8, 0.5, A, None) == ERR_ARG
    assert f(A, 4, 8, float("nan"), A, None) == ERR_ARG
    assert f(A, 4, 8, float("inf"), A, None) == ERR_ARG
    assert f(MIS, 4, 8, 0.5, A, None) == ERR_ALIGN


def test_workspace_size(lib):
    ws = lib.w4a16_gemm_workspace_size
    assert ws(1, 8192, 8192, 128) > 8192 * 4
    assert ws(4, 100, 256, 128) >= 4 * 100 * 4
    assert ws(0, 8, 128, 128) == 0
    # M above one launch's 128 tokens runs in chunks on the M = 128 workspace
    assert ws(300, 8, 128, 128) == ws(256, 8, 128, 128) > ws(128, 8, 128, 128) > ws(64, 8, 128, 128)
    assert ws(1 << 20, 4096, 4096, 128) == 0
    assert ws(1, 8, 100, 128) == 0
    assert ws(1, 8, 128, 64) == 0


def test_gemm_validation(lib):
    g = lib.w4a16_gemm
    need = lib.w4a16_gemm_workspace_size(1, 64, 256, 128)
    assert g(None, A, A, A, 1, 64, 256, 128, A, B, need, None) == ERR_ARG
    assert g(A, A, A, A, 0, 64, 256, 128, A, B, need, None) == ERR_ARG
    assert g(A, A, A, A, 1, 64, 256, 64, A, B, need, None) == ERR_UNSUPPORTED
    assert g(A, A, A, A, 1, 64, 200, 128, A, B, need, None) == ERR_SHAPE
    assert g(A, A, A, A, 1 << 24, 64, 256, 128, A, B, need, None) == ERR_SHAPE
    assert g(MIS, A, A, A, 1, 64, 256, 128, A, B, need, None) == ERR_ALIGN
    assert g(A, A, A, A, 1, 64, 256, 128, MIS, B, need, None) == ERR_ALIGN
    assert g(A, A, A, A, 1, 64, 256, 128, A, None, need, None) == ERR_WORKSPACE
    assert g(A, A, A, A, 1, 64, 256, 128, A, B, need - 1, None) == ERR_WORKSPACE
    assert "workspace" in _err(lib)
    assert g(A, A, A, A, 1, 64, 256, 128, A, MIS, need, None) == ERR_ALIGN


def test_gemm_check_validation(lib):
    assert lib.w4a16_gemm_check(None, None) == ERR_ARG


def test_reference_product_validation(lib):
    rp = lib.awq_reference_product
    assert rp(None, A, 4, 8, 128, A, None) == ERR_ARG
    assert rp(A, A, 0, 8, 128, A, None) == ERR_ARG
    assert rp(A, A, (1 << 20) + 1, 8, 128, A, None) == ERR_SHAPE
    assert rp(MIS, A, 4, 8, 128, A, None) == ERR_ALIGN


def test_w4a8_validation(lib):
    assert lib.w4a8_quantize_weight(None, 8, 128, 128, A, A, A, A, None) == ERR_ARG
    assert lib.w4a8_quantize_weight(A, 8, 128, 64, A, A, A, A, None) == ERR_UNSUPPORTED
    assert lib.w4a8_quantize_weight(A, 8, 200, 128, A, A, A, A, None) == ERR_SHAPE
    assert lib.w4a8_quantize_weight(A, 8, 131072, 128, A, A, A, A, None) == ERR_SHAPE
    assert lib.w4a8_quantize_act(A, 0, 128, A, A, None) == ERR_ARG
    assert lib.w4a8_quantize_act(A, 70000, 128, A, A, None) == ERR_SHAPE
    assert lib.w4a8_gemm_workspace_size(1, 8, 200, 128) == 0
    assert lib.w4a8_gemm_workspace_size(4, 8, 128, 128) > 0
    g = lib.w4a8_gemm
    assert g(A, A, A, A, A, A, 1, 8, 128, 128, A, None, None, 0, None) == ERR_WORKSPACE
    assert g(A, A, A, A, A, A, 1, 8, 128, 128, None, None, A, 1 << 20, None) == ERR_ARG
    assert g(A, A, A, A, A, A, 1, 8, 128, 128, A, MIS, A, 1 << 20, None) == ERR_ALIGN
    assert "w4a8_gemm" in _err(lib)


def test_noalloc_timeout_selftest_validation(lib):
    assert lib.w4a16_gemv_noalloc_timeout_selftest(0, None) == ERR_ARG
    assert lib.w4a16_gemv_noalloc_timeout_selftest(1000001, None) == ERR_ARG
    assert "limit_us" in _err(lib)


def test_wait_timeout_selftest_validation(lib):
    """Argument checks happen before any launch (no GPU needed)."""
    assert lib.w4a16_wait_timeout_selftest(None, 1000, None) == ERR_ARG
    buf = ctypes.create_string_buffer(64)
    addr = (ctypes.addressof(buf) + 15) & ~15
    assert lib.w4a16_wait_timeout_selftest(ctypes.c_void_p(addr + 4), 1000, None) == ERR_ARG  # misaligned
    assert lib.w4a16_wait_timeout_selftest(ctypes.c_void_p(addr), 0, None) == ERR_ARG
    assert lib.w4a16_wait_timeout_selftest(ctypes.c_void_p(addr), 1000001, None) == ERR_ARG


def test_python_binding_rejects_cpu_tensors():
    import torch
    with pytest.raises(w4.W4A16Error):
        w4.awq_quantize_pack(torch.zeros((8, 128), dtype=torch.float16))
    with pytest.raises(w4.W4A16Error):
        w4.w4a16_gemm(torch.zeros((1, 128), dtype=torch.float16), torch.zeros((8, 16), dtype=torch.int32),
                      torch.zeros((8, 1), dtype=torch.float16), torch.zeros((8, 1), dtype=torch.float16))


def test_search_workspace_size(lib):
    ws = lib.awq_search_workspace_size
    n = ws(11008, 4096, 512, 20, 128)
    # at least the packed weight, the divided tokens, the fp16 and fp32 outputs
    assert n >= 11008 * 4096 // 2 + 512 * 4096 * 2 + 512 * 11008 * (2 + 4)
    assert ws(256, 1024, 100, 11, 128) > 0
    assert ws(0, 1024, 100, 11, 128) == 0
    assert ws(256, 1000, 100, 11, 128) == 0
    assert ws(256, 1024, 0, 11, 128) == 0
    assert ws(256, 1024, 100, 0, 128) == 0
    assert ws(256, 1024, 100, 4097, 128) == 0
    assert ws(256, 1024, 100, 11, 64) == 0
    assert ws(1 << 20, 1 << 12, 1, 1, 128) == 0
    assert ws(1, 128, (1 << 20) + 1, 1, 128) == 0


def test_search_validation(lib):
    """Every rejection happens before anything is enqueued (no GPU needed)."""
    f = lib.awq_search_alpha
    grid = (ctypes.c_double * 3)(0.0, 0.5, 1.0)
    bad = (ctypes.c_double * 3)(0.0, float("nan"), 1.0)
    losses = (ctypes.c_double * 3)()
    best = ctypes.c_int(-1)
    need = lib.awq_search_workspace_size(64, 256, 10, 3, 128)

    def call(W=A, X=A, N=64, K=256, T=10, alphas=grid, n=3, group=128, bits=4, mode=0, out=losses, ws=B,
             nbytes=need):
        return f(W, X, N, K, T, alphas, n, group, bits, mode, out, ctypes.byref(best), ws, nbytes, None)

    assert call(W=None) == ERR_ARG
    assert call(alphas=None) == ERR_ARG
    assert call(out=None) == ERR_ARG
    assert call(ws=None) == ERR_ARG
    assert call(T=0) == ERR_ARG
    assert call(T=(1 << 20) + 1, K=128) == ERR_SHAPE
    assert call(n=0) == ERR_ARG
    assert call(n=5000) == ERR_ARG
    assert call(alphas=bad) == ERR_ARG
    assert "alphas[1]" in _err(lib)
    assert call(mode=3) == ERR_ARG
    assert call(group=64) == ERR_UNSUPPORTED
    assert call(bits=8) == ERR_UNSUPPORTED
    assert call(K=200) == ERR_SHAPE
    assert call(N=1 << 20, K=1 << 12) == ERR_SHAPE
    assert call(X=MIS) == ERR_ALIGN
    assert call(ws=MIS) == ERR_ALIGN
    assert call(nbytes=need - 1) == ERR_WORKSPACE
    assert "workspace" in _err(lib)
    assert best.value == -1


def test_gptq_validation(lib):
    """Every rejection happens before anything is enqueued (no GPU needed)."""
    h = lib.gptq_hessian
    assert h(None, 10, 128, 0.01, A, None) == ERR_ARG
    assert h(A, 0, 128, 0.01, A, None) == ERR_ARG
    assert h(A, 10, 128, -1.0, A, None) == ERR_ARG
    assert h(A, 10, 128, float("nan"), A, None) == ERR_ARG
    assert h(A, 10, 32768 + 128, 0.01, A, None) == ERR_SHAPE
    assert h(MIS, 10, 128, 0.01, A, None) == ERR_ALIGN
    ws = lib.gptq_sweep_workspace_size
    assert ws(100, 256, 128) >= 100 * 256 * 9
    assert ws(100, 200, 128) == 0 and ws(100, 256, 64) == 0 and ws(0, 256, 128) == 0
    assert ws(1, 32768 + 128, 128) == 0
    f = lib.gptq_sweep
    need = ws(64, 256, 128)
    assert f(None, A, 64, 256, 128, 4, 0, A, A, A, B, need, None) == ERR_ARG
    assert f(A, A, 64, 256, 128, 4, 5, A, A, A, B, need, None) == ERR_ARG
    assert f(A, A, 64, 256, 64, 4, 0, A, A, A, B, need, None) == ERR_UNSUPPORTED
    assert f(A, A, 64, 256, 128, 2, 0, A, A, A, B, need, None) == ERR_UNSUPPORTED
    assert f(A, A, 64, 200, 128, 4, 0, A, A, A, B, need, None) == ERR_SHAPE
    assert f(A, MIS, 64, 256, 128, 4, 0, A, A, A, B, need, None) == ERR_ALIGN
    assert f(A, A, 64, 256, 128, 4, 0, A, A, A, B, need - 1, None) == ERR_WORKSPACE


def test_gptq_factor_and_quantize_validation(lib):
    """Every rejection happens before anything is enqueued (no GPU needed)."""
    fws = lib.gptq_factor_workspace_size
    assert fws(4096) >= 2 * 4096 * 4096 * 8 and fws(0) == 0 and fws(32768 + 1) == 0
    f = lib.gptq_factor
    assert f(None, 256, A, B, fws(256), None) == ERR_ARG
    assert f(A, 0, A, B, fws(256), None) == ERR_ARG
    assert f(A, 40000, A, B, 1 << 40, None) == ERR_SHAPE
    assert f(MIS, 256, A, B, fws(256), None) == ERR_ALIGN
    assert f(A, 256, A, B, fws(256) - 1, None) == ERR_WORKSPACE
    qws = lib.gptq_quantize_workspace_size
    assert qws(64, 256, 128) > fws(256) + lib.gptq_sweep_workspace_size(64, 256, 128)
    assert qws(64, 200, 128) == 0 and qws(64, 256, 64) == 0
    q = lib.gptq_quantize
    need = qws(64, 256, 128)

    def call(W=A, X=A, N=64, K=256, T=10, damp=0.01, group=128, bits=4, mode=0, ws=B, nbytes=need):
        return q(W, X, N, K, T, damp, group, bits, mode, A, A, A, ws, nbytes, None)

    assert call(X=None) == ERR_ARG
    assert call(T=0) == ERR_ARG
    assert call(damp=float("inf")) == ERR_ARG
    assert call(mode=2) == ERR_ARG
    assert call(group=32) == ERR_UNSUPPORTED
    assert call(bits=5) == ERR_UNSUPPORTED
    assert call(K=200) == ERR_SHAPE
    assert call(X=MIS) == ERR_ALIGN
    assert call(nbytes=need - 1) == ERR_WORKSPACE


def test_python_binding_rejects_cpu_tensors_for_search_and_gptq():
    """No CPU fallback: every binding refuses host tensors before calling the library."""
    import torch
    W = torch.zeros((8, 128), dtype=torch.float16)
    X = torch.zeros((4, 128), dtype=torch.float16)
    H = torch.eye(128, dtype=torch.float64)
    with pytest.raises(w4.W4A16Error):
        w4.awq_search_alpha(W, X, [0.0, 0.5])
    with pytest.raises(w4.W4A16Error):
        w4.gptq_hessian(X)
    with pytest.raises(w4.W4A16Error):
        w4.gptq_sweep(W, H)
    with pytest.raises(w4.W4A16Error):
        w4.gptq_factor(H)
    with pytest.raises(w4.W4A16Error):
        w4.gptq_quantize(W, X)
