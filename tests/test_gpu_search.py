"""Parity of the AWQ alpha search (awq_search_alpha) with the CPU oracle.

L(alpha) = mean over outputs of (Q(W s)(s^-1 X) - W X)^2, s = s_X^alpha, and
alpha* = argmin over the grid ("MIT 6.5940 Fall 2024 Lecture 13: LLM
Deployment" reading guide, §AWQ, slide 28).  The codes behind every loss are
bit-exact to the oracle's (the quantizer's own tests pin that); the losses
differ only through the W4A16 GEMM's fp32 accumulation (and, on the tensor
cores, the fp16 rounding of w_hat before the MMA) and through the fp32
target.  Those errors are far below the quantization error and not
correlated with it, so each loss must agree to RTOL relative; the GEMM's
stated worst-case bound would allow much more, but it is not what decides
alpha.  Where the two searches pick different grid points, the oracle's loss
at the GPU's choice must be within RTOL of its own minimum.
"""
import numpy as np
import pytest
import torch

import oracle
import w4a16_decode_gemv_b200 as w4
from w4a16_decode_gemv_b200 import build, inputs

pytestmark = pytest.mark.gpu

RTOL = 5e-3


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()
    w4.load_library()
    return torch.device("cuda:0")


def to_dev(a, dev):
    return torch.from_numpy(np.ascontiguousarray(a)).to(dev)


def compare(losses, best, ref_losses, ref_best):
    losses, ref = np.asarray(losses), np.asarray(ref_losses)
    rel = np.abs(losses - ref) / ref
    assert np.all(rel <= RTOL), f"relative loss differences {rel}"
    assert best == int(np.argmin(losses))
    if best != ref_best:
        assert ref[best] <= ref[ref_best] * (1 + RTOL)


@pytest.mark.parametrize("N,K,T,bits,mode", [
    (256, 1024, 100, 4, oracle.ASYM),   # one GEMM launch with a 128-token tile
    (129, 512, 130, 4, oracle.ASYM),    # odd N, chunks of 128 + 2 tokens (a GEMV tail)
    (200, 512, 300, 3, oracle.SYM),     # the 3-bit symmetric codes, chunks of 128 + 128 + 44
    (300, 256, 3, 4, oracle.ASYM),      # a few tokens: the CUDA-core GEMV only
    (64, 128, 1, 4, oracle.ASYM),       # one token, one group
])
def test_search_small(dev, N, K, T, bits, mode):
    W, X = inputs.random_case(N * 31 + T, N, K, T)
    alphas = np.linspace(0.0, 1.0, 11)
    ref_losses, ref_best = oracle.awq_search(W, X, alphas, 128, bits, mode)
    losses, best = w4.awq_search_alpha(to_dev(W, dev), to_dev(X, dev), alphas, bits=bits, mode=mode)
    compare(losses, best, ref_losses, ref_best)


def test_search_repeatable_and_grid_order(dev):
    """The same call gives identical losses; a permuted grid permutes them."""
    W, X = inputs.random_case(17, 256, 1024, 96)
    Wd, Xd = to_dev(W, dev), to_dev(X, dev)
    alphas = [0.0, 0.25, 0.5, 0.75, 1.0]
    l1, b1 = w4.awq_search_alpha(Wd, Xd, alphas)
    l2, b2 = w4.awq_search_alpha(Wd, Xd, alphas)
    assert l1 == l2 and b1 == b2
    l3, _ = w4.awq_search_alpha(Wd, Xd, alphas[::-1])
    assert l3 == l1[::-1]


def test_search_workspace_reused_with_garbage(dev):
    """The workspace is scratch: a buffer full of 0xFF gives the same losses."""
    W, X = inputs.random_case(23, 192, 512, 70)
    Wd, Xd = to_dev(W, dev), to_dev(X, dev)
    alphas = [0.0, 0.5, 1.0]
    ws = torch.full((w4.search_workspace_size(192, 512, 70, 3),), 255, dtype=torch.uint8, device=dev)
    l1, _ = w4.awq_search_alpha(Wd, Xd, alphas, workspace=ws)
    l2, _ = w4.awq_search_alpha(Wd, Xd, alphas)
    assert l1 == l2


def test_search_alpha_zero_is_plain_rtn(dev):
    """alpha = 0 gives s = 1: the loss is that of plain RTN codes with the undivided activation."""
    W, X = inputs.random_case(29, 128, 512, 20)
    (l0,), _ = w4.awq_search_alpha(to_dev(W, dev), to_dev(X, dev), [0.0])
    q, sc, z = oracle.quantize_pack(W, None)
    y_q = (X.astype(np.float64) @ oracle.dequant(q, sc, z).T).astype(np.float16).astype(np.float64)
    y = X.astype(np.float64) @ W.astype(np.float64).T
    ref = float(np.mean((y_q - y) ** 2))
    assert abs(l0 - ref) <= RTOL * ref


def test_search_calibration_workload(dev):
    """The 11008 x 4096 layer and its 512 calibration tokens with a 20-point grid, the
    search the bench times; the oracle checks the ends, alpha = 0.5 and the GPU's choice
    with its neighbours."""
    W, X, _ = inputs.quant_workload()
    alphas = np.arange(20) / 19.0
    losses, best = w4.awq_search_alpha(to_dev(W, dev), to_dev(X, dev), alphas)
    assert best == int(np.argmin(losses))
    check = sorted({0, 19, 10, best, max(best - 1, 0), min(best + 1, 19)})
    ref = {i: oracle.awq_loss(W, X, float(alphas[i])) for i in check}
    for i in check:
        assert abs(losses[i] - ref[i]) <= RTOL * ref[i], (i, losses[i], ref[i])
    for i in check:
        assert ref[best] <= ref[i] * (1 + RTOL)
