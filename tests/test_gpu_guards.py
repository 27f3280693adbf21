"""Stray stores, checked without a sanitizer: guard regions around y and the workspace.

Every kernel writes y and its workspace through computed indices; a ragged
shape (N not a multiple of the row tile, M not a multiple of the token tile,
K / 128 odd or not a multiple of 4) is where an index can run past its
buffer.  Here y and the workspace are views at the start of larger buffers
whose remainder holds a fixed bit pattern; after the call the pattern must be
untouched, the outputs must match the oracle, and the part of the workspace
that must start at zero must be zero again.  (A memory checker is not
available for these runs; this covers what it would catch in the outputs and
the workspace.)  The same guards are kept around the W4A8 product, and the
alpha search's target product is checked element by element against the
oracle's exact X W^T.
"""
import numpy as np
import pytest
import torch

import oracle
import w4a16_decode_gemv_b200 as w4
from w4a16_decode_gemv_b200 import build, inputs

pytestmark = pytest.mark.gpu

GUARD = 4096          # elements of guard after y, bytes after the workspace
PATTERN = 0x5A3C      # fp16 bit pattern in y's guard
PATTERN_B = 0xA5      # byte pattern in the workspace's guard


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()
    w4.load_library()
    return torch.device("cuda:0")


def to_dev(a, dev):
    return torch.from_numpy(np.ascontiguousarray(a)).to(dev)


def guarded_y(M, N, dev):
    buf = torch.full((M * N + GUARD,), PATTERN, dtype=torch.int16, device=dev)
    return buf, buf[:M * N].view(torch.float16).view(M, N)


def guarded_ws(need, dev):
    buf = torch.full((need + GUARD,), PATTERN_B, dtype=torch.uint8, device=dev)
    buf[:need].zero_()
    return buf, buf[:need]


@pytest.mark.parametrize("M,N,K", [
    (1, 17, 1152), (1, 300, 4096), (2, 513, 1152), (3, 300, 11008), (4, 17, 22016),
    (5, 17, 1152), (16, 300, 1152), (40, 513, 4096), (129, 300, 1024), (200, 17, 2048), (300, 513, 1152),
])
def test_w4a16_gemm_stays_inside_y_and_workspace(dev, M, N, K):
    W, x = inputs.random_case(M * 31 + N, N, K, M)
    qo, so, zo = oracle.quantize_pack(W, None, 128, 4, oracle.ASYM)
    ybuf, y = guarded_y(M, N, dev)
    need = w4.gemm_workspace_size(M, N, K)
    wbuf, ws = guarded_ws(need, dev)
    w4.w4a16_gemm(to_dev(x, dev), to_dev(qo.view(np.int32), dev), to_dev(so, dev), to_dev(zo, dev), out=y,
                  workspace=ws)
    w4.gemm_check(ws)
    assert bool((ybuf[M * N:] == PATTERN).all()), "a store past the end of y"
    assert bool((wbuf[need:] == PATTERN_B).all()), "a store past the end of the workspace"
    # what must start at zero is left zero: the status word, flags, counters and GEMV partials
    assert int(ws[:w4.gemm_workspace_size(min(M, 4), N, K)].count_nonzero()) == 0
    y_ref, B = oracle.gemm(x, qo, so, zo)
    assert np.all(np.abs(y.cpu().numpy().astype(np.float64) - y_ref) <= 2e-3 * B + 1e-3)


@pytest.mark.parametrize("M,N,K", [(1, 17, 1152), (3, 300, 11008), (5, 513, 1152), (64, 17, 4096), (200, 300, 1024)])
def test_w4a8_gemm_stays_inside_y_and_workspace(dev, M, N, K):
    W, x = inputs.random_case(M * 37 + N, N, K, M)
    qo, s1o, s2o, zso = oracle.w4a8_quantize_weight(W)
    x8o, sxo = oracle.w4a8_quantize_act(x)
    ybuf, y = guarded_y(M, N, dev)
    abuf = torch.full((M * N + GUARD,), 0x5A5A5A5A, dtype=torch.int32, device=dev)
    need = w4.w4a8_gemm_workspace_size(M, N, K)
    wbuf, ws = guarded_ws(need, dev)
    args = [to_dev(a, dev) for a in (x8o, sxo, qo.view(np.int32), s1o, s2o, zso)]
    w4.w4a8_gemm(*args, out=y, acc=abuf[:M * N].view(M, N), workspace=ws)
    w4.gemm_check(ws)
    assert bool((ybuf[M * N:] == PATTERN).all()), "a store past the end of y"
    assert bool((abuf[M * N:] == 0x5A5A5A5A).all()), "a store past the end of acc"
    assert bool((wbuf[need:] == PATTERN_B).all()), "a store past the end of the workspace"
    yo, acco = oracle.w4a8_gemm(x8o, sxo, qo, s1o, s2o, zso)
    assert np.array_equal(abuf[:M * N].view(M, N).cpu().numpy().astype(np.int64), acco)
    assert np.array_equal(y.cpu().numpy().view(np.uint16), yo.view(np.uint16))


@pytest.mark.parametrize("N,K,T", [(300, 1152, 7), (1000, 4096, 64), (64, 11008, 130)])
def test_search_target_product_matches_exact(dev, N, K, T):
    """The alpha search measures against y = X W^T formed in fp32 from exact fp16
    products in k order; every element lies within K fp32 roundings of the exact sum."""
    W, _ = inputs.random_case(N + K, N, K, 1)
    rng = np.random.default_rng(T)
    X = inputs.activations(rng, T, K, inputs.outlier_channels(rng, K))
    Y = w4.awq_reference_product(to_dev(X, dev), to_dev(W, dev)).cpu().numpy().astype(np.float64)
    Xf, Wf = X.astype(np.float64), W.astype(np.float64)
    exact = Xf @ Wf.T
    bound = np.abs(Xf) @ np.abs(Wf).T
    assert np.all(np.abs(Y - exact) <= K * 2.0 ** -24 * bound + 1e-30)
