"""Parity of the W4A8 path (progressive group quantization) with the CPU oracle.

"MIT 6.5940 Fall 2024 Lecture 13" reading guide, §QServe: every result here is
decided by integers or by one rounding of an exactly known value, so the GPU
must agree with the oracle bit for bit: the packed codes, s1, s2 and zs of
the weight quantizer, x8 and s_x of the activation quantizer, the exact int32
accumulators of the product and y = fp16((acc * s_x) * s1).
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


def to_dev(a, dev):
    return torch.from_numpy(np.ascontiguousarray(a)).to(dev)


def bits(a):
    a = np.ascontiguousarray(a)
    return a.view(np.uint16) if a.dtype == np.float16 else a


def quantize_both(W, dev):
    q, s1, s2, zs = (t.cpu().numpy() for t in w4.w4a8_quantize_weight(to_dev(W, dev)))
    qo, s1o, s2o, zso = oracle.w4a8_quantize_weight(W)
    assert np.array_equal(q.view(np.uint32), qo)
    assert np.array_equal(bits(s1), bits(s1o))
    assert np.array_equal(s2, s2o)
    assert np.array_equal(zs, zso)
    return qo, s1o, s2o, zso


@pytest.mark.parametrize("N,K,sigma,seed", [
    (8, 128, 0.02, 0),
    (300, 1152, 0.02, 1),
    (1000, 4096, 0.5, 2),
    (17, 22016, 0.015, 3),
])
def test_w4a8_weight_quantizer_bit_exact(dev, N, K, sigma, seed):
    W, _ = inputs.random_case(seed, N, K, 1, sigma=sigma)
    quantize_both(W, dev)


def test_w4a8_weight_quantizer_edge_rows(dev):
    """Zero rows (s1 = fp16(1/119)), rows of one value, exact level-1 ties, tiny and
    huge magnitudes, and groups that lie entirely on one side of zero."""
    rng = np.random.default_rng(9)
    K = 512
    W = (rng.standard_normal((12, K)) * 0.02).astype(np.float16)
    W[0] = 0
    W[1] = np.float16(0.5)
    W[2, :128] = np.float16(3.0)          # a group of one positive value
    W[3, 128:256] = -np.abs(W[3, 128:256])  # a group all below zero
    W[4] = np.float16(6e-8)               # subnormal magnitudes
    W[5] = np.clip(rng.standard_normal(K) * 2e4, -65000, 65000).astype(np.float16)  # large, finite
    W[6, ::2] = np.float16(119.0)         # s1 = 1: every w8 an integer
    W[6, 1::2] = np.arange(-59, 197, dtype=np.float16)[:K // 2] / 2  # half-integer quotients: ties
    W[7, 0] = np.float16(-119.0)
    quantize_both(W, dev)


@pytest.mark.parametrize("M,K,seed", [(1, 128, 0), (3, 4096, 1), (64, 8192, 2), (300, 1152, 3)])
def test_w4a8_activation_quantizer_bit_exact(dev, M, K, seed):
    _, x = inputs.random_case(seed, 8, K, M)
    x[0, :] = 0 if M > 2 else x[0, :]
    x8, sx = (t.cpu().numpy() for t in w4.w4a8_quantize_act(to_dev(x, dev)))
    x8o, sxo = oracle.w4a8_quantize_act(x)
    assert np.array_equal(x8, x8o)
    assert np.array_equal(bits(sx), bits(sxo))


def test_w4a8_activation_quantizer_every_fp16(dev):
    """Every finite fp16 value against a few token scales (the rounding of the quotient)."""
    vals = np.arange(65536, dtype=np.uint16).view(np.float16)
    vals = vals[np.isfinite(vals)]
    rows = []
    for amax in (np.float16(1.0), np.float16(127.0), np.float16(0.3), np.float16(65504.0)):
        sel = vals[np.abs(vals.astype(np.float64)) <= float(amax)]
        row = np.zeros(64512, dtype=np.float16)
        row[:sel.size] = sel
        row[-1] = amax
        rows.append(row)
    x = np.stack(rows)
    x8, sx = (t.cpu().numpy() for t in w4.w4a8_quantize_act(to_dev(x, dev)))
    x8o, sxo = oracle.w4a8_quantize_act(x)
    assert np.array_equal(bits(sx), bits(sxo))
    assert np.array_equal(x8, x8o)


def _gemm_case(dev, M, N, K, seed, sigma=0.02):
    W, x = inputs.random_case(seed, N, K, M, sigma=sigma)
    qo, s1o, s2o, zso = oracle.w4a8_quantize_weight(W)
    x8o, sxo = oracle.w4a8_quantize_act(x)
    args = [to_dev(a, dev) for a in (x8o, sxo, qo.view(np.int32), s1o, s2o, zso)]
    y, acc = w4.w4a8_gemm(*args, acc=True)
    yo, acco = oracle.w4a8_gemm(x8o, sxo, qo, s1o, s2o, zso)
    assert np.array_equal(acc.cpu().numpy().astype(np.int64), acco)
    assert np.array_equal(bits(y.cpu().numpy()), bits(yo))
    return args, yo


@pytest.mark.parametrize("M,N,K", [
    (1, 1, 512),        # one row
    (1, 300, 1024),     # ragged row block, K = half a unit
    (1, 4096, 4096),
    (2, 513, 2048),
    (3, 1000, 11008),   # 86 groups: units past the last group
    (4, 256, 8192),
    (4, 64, 22016),     # 172 groups per row
])
def test_w4a8_gemv_exact(dev, M, N, K):
    _gemm_case(dev, M, N, K, seed=M * 7919 + N)


def test_w4a8_gemv_workload_rows(dev):
    """The K = N = 8192 skinny layer at M = 1 and 4 (the bench's launch), every output exact."""
    (layer,) = inputs.layer_set(inputs.SKINNY)
    qg, s1g, s2g, zsg = w4.w4a8_quantize_weight(to_dev(layer.W, dev))
    for M in (1, 4):
        x8, sx = w4.w4a8_quantize_act(to_dev(layer.x[:M], dev))
        y, acc = w4.w4a8_gemm(x8, sx, qg, s1g, s2g, zsg, acc=True)
        rows = np.unique(np.concatenate([np.random.default_rng(M).choice(layer.N, 252, replace=False),
                                         [0, 255, 256, layer.N - 1]]))
        qo, s1o, s2o, zso = oracle.w4a8_quantize_weight(layer.W[rows])
        assert np.array_equal(qg.cpu().numpy().view(np.uint32)[rows], qo)
        x8o, sxo = oracle.w4a8_quantize_act(layer.x[:M])
        yo, acco = oracle.w4a8_gemm(x8o, sxo, qo, s1o, s2o, zso)
        assert np.array_equal(acc.cpu().numpy()[:, rows].astype(np.int64), acco)
        assert np.array_equal(bits(y.cpu().numpy()[:, rows]), bits(yo))


def test_w4a8_gemv_repeats_bit_for_bit(dev):
    args, yo = _gemm_case(dev, 2, 700, 4096, seed=5)
    for _ in range(3):
        assert np.array_equal(bits(w4.w4a8_gemm(*args).cpu().numpy()), bits(yo))


@pytest.mark.parametrize("M,N,K", [
    (5, 300, 1024),      # token tile 16, ragged row tile
    (16, 513, 1152),     # 9 groups: the last unit of a row holds one group
    (33, 1000, 11008),   # 86 groups (two past the last unit), token tile 64
    (64, 2048, 256),     # one unit per row
    (100, 256, 2048),    # token tile 128
    (150, 300, 4096),    # token tile 192
    (200, 384, 4096),    # token tile 256
    (300, 256, 8192),    # 256 + 44 tokens
])
def test_w4a8_tensor_core_exact(dev, M, N, K):
    _gemm_case(dev, M, N, K, seed=M * 104729 + N)


def test_w4a8_tensor_core_workload_rows(dev):
    """K = N = 8192 at M = 16 and 64 (the bench's launches): sampled rows exact."""
    (layer,) = inputs.layer_set(inputs.SKINNY)
    qg, s1g, s2g, zsg = w4.w4a8_quantize_weight(to_dev(layer.W, dev))
    rows = np.unique(np.concatenate([np.random.default_rng(64).choice(layer.N, 252, replace=False),
                                     [0, 127, 128, layer.N - 1]]))
    qo, s1o, s2o, zso = oracle.w4a8_quantize_weight(layer.W[rows])
    for M in (16, 64):
        x8, sx = w4.w4a8_quantize_act(to_dev(layer.x[:M], dev))
        y, acc = w4.w4a8_gemm(x8, sx, qg, s1g, s2g, zsg, acc=True)
        x8o, sxo = oracle.w4a8_quantize_act(layer.x[:M])
        yo, acco = oracle.w4a8_gemm(x8o, sxo, qo, s1o, s2o, zso)
        assert np.array_equal(acc.cpu().numpy()[:, rows].astype(np.int64), acco)
        assert np.array_equal(bits(y.cpu().numpy()[:, rows]), bits(yo))
