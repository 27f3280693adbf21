"""GPTQ end to end on the GPU: gptq_factor and gptq_quantize against the oracle.

G = Cholesky(H^-1)^T ("CMU 11-868 LLM Systems: Model Quantization" reading
guide, §L20 "GPTQ", step 1) is computed on the GPU by a reversed-order
Cholesky and a triangular inverse whose sums run over warp lanes, so it agrees
with numpy's to rounding.  Given G, the sweep is bit-exact (test_gpu_gptq.py);
with the GPU's own G the codes can differ from the oracle's only where a swept
value lies within about 1e-12 of a rounding boundary, which random data almost
never reaches: at least 99.9 % of the codes must agree, and the layer's output
error must match the oracle's to 1e-6.
(This file runs after the other GPU tests: it covers the whole pipeline.)
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


@pytest.mark.parametrize("K,T", [(128, 200), (384, 300), (1024, 512)])
def test_factor(dev, K, T):
    _, X = inputs.random_case(K + T, 8, K, T)
    H = oracle.gptq_hessian(X)
    G = w4.gptq_factor(to_dev(H, dev)).cpu().numpy()
    ref = oracle.gptq_factor(H)
    assert np.array_equal(G, np.triu(G))
    assert np.abs(G - ref).max() <= 1e-10 * np.abs(ref).max()


def _output_error(W, X, q, s, z):
    e = W.astype(np.float64) - oracle.dequant(q, s, z)
    return float(np.sum((e @ X.astype(np.float64).T) ** 2))


@pytest.mark.parametrize("N,K,bits,mode", [(96, 256, 4, oracle.ASYM), (64, 384, 3, oracle.SYM)])
def test_quantize_small(dev, N, K, bits, mode):
    rng = np.random.default_rng(N + K)
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float16)
    z0 = rng.standard_normal((2 * K, K))
    X = (z0 @ (np.eye(K) + 0.8 * rng.standard_normal((K, K)) / math.sqrt(K))).astype(np.float16)
    q, s, z = w4.gptq_quantize(to_dev(W, dev), to_dev(X, dev), bits=bits, mode=mode)
    qo, so, zo = oracle.gptq_quantize(W, X, 128, bits, mode)
    q, s, z = q.cpu().numpy().view(np.uint32), s.cpu().numpy(), z.cpu().numpy()
    assert (oracle.unpack_v1(q) == oracle.unpack_v1(qo)).mean() >= 0.999
    e_gpu, e_or = _output_error(W, X, q, s, z), _output_error(W, X, qo, so, zo)
    assert abs(e_gpu - e_or) <= 1e-6 * e_or


def test_quantize_calibration_workload_sampled_rows(dev):
    """The 11008 x 4096 layer with its 512 calibration tokens, Hessian, factor and sweep all
    on the GPU; 24 sampled rows against the oracle's GPTQ."""
    W, X, _ = inputs.quant_workload()
    q, s, z = w4.gptq_quantize(to_dev(W, dev), to_dev(X, dev))
    rows = np.random.default_rng(4).choice(W.shape[0], 24, replace=False)
    qo, so, zo = oracle.gptq_quantize(W[rows], X)
    same = (oracle.unpack_v1(q.cpu().numpy().view(np.uint32)[rows]) == oracle.unpack_v1(qo)).mean()
    assert same >= 0.999
