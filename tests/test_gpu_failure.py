"""Failure detection on the GPU without a fault: a bounded wait that runs out.

The GEMM kernels bound every barrier wait by the device clock; a wait that
gives up sets the workspace status word, and w4a16_gemm_check reports it.  The
self-test kernel takes that path on a barrier nothing completes; afterwards the
context and the workspace stay usable.
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


def test_wait_timeout_reported_then_cleared(dev):
    N, K = 256, 1024
    ws = torch.zeros(w4.gemm_workspace_size(1, N, K), dtype=torch.uint8, device=dev)
    w4.wait_timeout_selftest(ws, limit_us=2000)
    with pytest.raises(w4.W4A16Error, match="gave up waiting"):
        w4.gemm_check(ws)
    w4.gemm_check(ws)  # the check cleared the status word
    # the context and the workspace are still good for a GEMV
    W, x = inputs.random_case(3, N, K, 1)
    qo, so, zo = oracle.quantize_pack(W, None, 128, 4, oracle.ASYM)
    y = w4.w4a16_gemm(torch.from_numpy(x).to(dev), torch.from_numpy(qo.view(np.int32)).to(dev),
                      torch.from_numpy(so).to(dev), torch.from_numpy(zo).to(dev), workspace=ws)
    w4.gemm_check(ws)
    y_ref, B = oracle.gemm(x, qo, so, zo)
    assert np.all(np.abs(y.cpu().numpy().astype(np.float64) - y_ref) <= 2e-3 * B + 1e-3)
