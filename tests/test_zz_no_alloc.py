"""w4a16_gemv_noalloc, the allocation-free GEMV entry point, against w4a16_gemm.

Some callers cannot allocate device memory (fixed-budget servers, plug-ins
without an allocator), so the library offers a GEMV that keeps its scratch in
a fixed device array.  This file checks, through the C ABI, that two calls in
a row give the same output as the regular entry point within the tolerance of
the other GEMV tests.  It is named to be collected last, and passes both alone
and after the other tests.
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


@pytest.mark.parametrize("M,N,K", [(1, 4096, 4096), (3, 1000, 11008), (4, 8192, 2048)])
def test_noalloc_matches_regular_entry_point_twice(dev, M, N, K):
    W, x = inputs.random_case(7 * N + M, N, K, M)
    qo, so, zo = oracle.quantize_pack(W, None, 128, 4, oracle.ASYM)
    args = [torch.from_numpy(a).to(dev) for a in (x, qo.view(np.int32), so, zo)]
    y_ref = w4.w4a16_gemm(*args).cpu().numpy().astype(np.float64)
    _, B = oracle.gemm(x, qo, so, zo)
    tol = 2e-3 * B + 1e-3
    out = torch.empty((M, N), dtype=torch.float16, device=dev)
    for _ in range(2):
        out.fill_(float("nan"))
        y = w4.w4a16_gemv_noalloc(*args, out=out)
        torch.cuda.synchronize()
        diff = np.abs(y.cpu().numpy().astype(np.float64) - y_ref)
        assert np.all(np.isfinite(diff))
        assert np.all(diff <= tol)


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
