"""GPTQ on the GPU (gptq_hessian, gptq_sweep) against the CPU oracle.

The sweep is defined operation by operation in fp64 ("CMU 11-868 LLM Systems:
Model Quantization" reading guide, §L20 "GPTQ"; the order is stated in
include/w4a16.h), so given the same factor G its codes, steps and zero points
must be bit-exact to oracle.gptq_sweep.  G is the oracle's (numpy's Cholesky of
numpy's inverse of the oracle's H): the factorization itself is not on the GPU
yet.  The Hessian's entries are fp64 sums whose order differs from numpy's
matmul, so they are compared to 1e-12 relative.
"""
import math

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


def to_dev(a, dev):
    return torch.from_numpy(np.ascontiguousarray(a)).to(dev)


def correlated_tokens(seed, T, K):
    """Calibration tokens with correlated channels (a seeded random mixing), so that
    rounding errors really move between columns."""
    rng = np.random.default_rng(seed)
    z = rng.standard_normal((T, K))
    a = np.eye(K) + 0.8 * rng.standard_normal((K, K)) / math.sqrt(K)
    return (z @ a).astype(np.float16)


@pytest.mark.parametrize("T,K", [(100, 384), (37, 200), (512, 128)])
def test_hessian(dev, T, K):
    _, X = inputs.random_case(T * 7 + K, 8, K, T)
    H = w4.gptq_hessian(to_dev(X, dev)).cpu().numpy()
    ref = oracle.gptq_hessian(X)
    np.testing.assert_allclose(H, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())


def sweep_case(dev, N, K, bits, mode, seed):
    W, _ = inputs.random_case(seed, N, K, 1)
    X = correlated_tokens(seed, 3 * K // 2, K)
    G = oracle.gptq_factor(oracle.gptq_hessian(X))
    q, s, z = w4.gptq_sweep(to_dev(W, dev), to_dev(G, dev), bits=bits, mode=mode)
    u, d0, z0, _ = oracle.gptq_sweep(W, G, 128, bits, mode)
    assert np.array_equal(q.cpu().numpy().view(np.uint32), oracle.pack_v1(u))
    assert np.array_equal(s.cpu().numpy().view(np.uint16), d0.view(np.uint16))
    assert np.array_equal(z.cpu().numpy().view(np.uint16), z0.view(np.uint16))
    return W, q, s, z


@pytest.mark.parametrize("N,K,bits,mode", [
    (37, 128, 4, oracle.ASYM),     # one block: no update right of it
    (300, 384, 4, oracle.ASYM),    # ragged rows, three blocks
    (64, 512, 3, oracle.SYM),      # 3-bit symmetric groups
    (1, 256, 4, oracle.ASYM),      # one row
])
def test_sweep_bit_exact(dev, N, K, bits, mode):
    sweep_case(dev, N, K, bits, mode, seed=N + K)


def test_sweep_identity_factor_is_rtn(dev):
    """G = I / sqrt(c): no error moves, so the sweep gives awq_quantize_pack's codes."""
    W, _ = inputs.random_case(5, 96, 256, 1)
    G = np.eye(256) / 3.0
    q, s, z = w4.gptq_sweep(to_dev(W, dev), to_dev(G, dev))
    q0, s0, z0 = w4.awq_quantize_pack(to_dev(W, dev))
    assert torch.equal(q, q0) and torch.equal(s, s0) and torch.equal(z, z0)


def test_sweep_feeds_the_gemv(dev):
    """GPTQ's output is layout v1: w4a16_gemm on it agrees with the oracle's product."""
    W, q, s, z = sweep_case(dev, 200, 512, 4, oracle.ASYM, seed=9)
    _, x = inputs.random_case(10, 8, 512, 3)
    y = w4.w4a16_gemm(to_dev(x, dev), q, s, z).cpu().numpy().astype(np.float64)
    y_ref, B = oracle.gemm(x, q.cpu().numpy().view(np.uint32), s.cpu().numpy(), z.cpu().numpy())
    assert np.all(np.abs(y - y_ref) <= 2e-3 * B + 1e-3)


def test_sweep_calibration_workload_sampled_rows(dev):
    """The 11008 x 4096 layer with the Hessian of its 512 calibration tokens: the whole
    sweep on the GPU; rows are independent, so 24 sampled rows are swept by the oracle."""
    W, X, _ = inputs.quant_workload()
    G = oracle.gptq_factor(oracle.gptq_hessian(X))
    q, s, z = w4.gptq_sweep(to_dev(W, dev), to_dev(G, dev))
    rows = np.unique(np.concatenate([np.random.default_rng(4).choice(W.shape[0], 20, replace=False),
                                     [0, 1, 8191, W.shape[0] - 1]]))
    u, d0, z0, _ = oracle.gptq_sweep(W[rows], G)
    assert np.array_equal(q.cpu().numpy().view(np.uint32)[rows], oracle.pack_v1(u))
    assert np.array_equal(s.cpu().numpy().view(np.uint16)[rows], d0.view(np.uint16))
    assert np.array_equal(z.cpu().numpy().view(np.uint16)[rows], z0.view(np.uint16))
