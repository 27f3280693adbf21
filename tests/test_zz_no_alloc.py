"""w4a16_gemv_noalloc, the allocation-free GEMV entry point, against the oracle.

Some callers cannot allocate device memory: servers that reserve every buffer
at start-up, plug-ins handed only the tensors they work on, hosts without a
device allocator.  The library gives them a GEMV that keeps its scratch in a
fixed device array.  This file checks, through the C ABI, that two calls in a
row each match the oracle's exact product within the tolerance of the other
GEMV tests, that the two are identical bit for bit (the split-K reduction adds
at most two partial sums per output onto zero, which commute), and that a
timed-out wait in that path is reported by w4a16_gemv_noalloc_check.  It is named to be collected last, and
passes both alone and after the other tests.
"""
import numpy as np
import pytest
import torch

import oracle
import w4a16_decode_gemv_b200 as w4
from w4a16_decode_gemv_b200 import build, inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()
    w4.load_library()
    return torch.device("cuda:0")


def _case(dev, M, N, K):
    W, x = inputs.random_case(7 * N + M, N, K, M)
    qo, so, zo = oracle.quantize_pack(W, None, 128, 4, oracle.ASYM)
    args = [torch.from_numpy(a).to(dev) for a in (x, qo.view(np.int32), so, zo)]
    y_ref, B = oracle.gemm(x, qo, so, zo)
    return args, y_ref, 2e-3 * B + 1e-3


@pytest.mark.parametrize("M,N,K", [(1, 4096, 4096), (2, 3000, 1152), (3, 1000, 11008), (4, 8192, 2048)])
def test_noalloc_matches_oracle_twice(dev, M, N, K):
    args, y_ref, tol = _case(dev, M, N, K)
    out = torch.empty((M, N), dtype=torch.float16, device=dev)
    ys = []
    for _ in range(2):
        out.fill_(float("nan"))
        y = w4.w4a16_gemv_noalloc(*args, out=out)
        w4.gemv_noalloc_check(dev)
        yh = y.cpu().numpy()
        diff = np.abs(yh.astype(np.float64) - y_ref)
        assert np.all(np.isfinite(diff))
        assert np.all(diff <= tol)
        ys.append(yh)
    # at most two split-K partial sums per output, added onto zero: the same y
    assert np.array_equal(ys[0].view(np.uint16), ys[1].view(np.uint16))


def test_noalloc_timeout_is_reported_then_cleared(dev):
    w4.gemv_noalloc_timeout_selftest(limit_us=2000, device=dev)
    with pytest.raises(w4.W4A16Error, match="gave up waiting"):
        w4.gemv_noalloc_check(dev)
    w4.gemv_noalloc_check(dev)  # the check cleared the status word
    args, y_ref, tol = _case(dev, 2, 512, 1024)
    y = w4.w4a16_gemv_noalloc(*args)
    w4.gemv_noalloc_check(dev)
    assert np.all(np.abs(y.cpu().numpy().astype(np.float64) - y_ref) <= tol)


def test_noalloc_rejects_oversized_scratch(dev):
    lib = w4.load_library()
    cap = lib.w4a16_gemv_noalloc_max_scratch()
    assert cap == 512 * 1024
    N = cap // 4  # M=4 partial sums alone exceed the array
    with pytest.raises(w4.W4A16Error, match="scratch"):
        x = torch.zeros((4, 128), dtype=torch.float16, device=dev)
        q = torch.zeros((N, 16), dtype=torch.int32, device=dev)
        s = torch.zeros((N, 1), dtype=torch.float16, device=dev)
        w4.w4a16_gemv_noalloc(x, q, s, s)
