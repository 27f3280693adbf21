"""Parity of the tensor-core GEMM (M = 5..256 per launch, larger M in chunks of
256 tokens) with the CPU oracle.

Every case goes through the C ABI (``w4a16_gemm``).  The output must satisfy,
per element, |y - y_ref| <= 2e-3 * B + 1e-3 with B = sum_k |x * w_hat| and
y_ref the fp64 product with the oracle's dequantized weight.
"""
import numpy as np
import pytest
import torch

import oracle
import w4a16_decode_gemv_b200 as w4
from w4a16_decode_gemv_b200 import build, inputs

pytestmark = pytest.mark.gpu

RTOL, ATOL = 2e-3, 1e-3


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()
    w4.load_library()
    return torch.device("cuda:0")


def to_dev(a, dev):
    return torch.from_numpy(np.ascontiguousarray(a)).to(dev)


def check(y, x, qw, sc, zr, rows=None):
    if rows is None:
        y_ref, B = oracle.gemm(x, qw, sc, zr)
        y = y.astype(np.float64)
    else:
        y_ref, B = oracle.gemm_rows(x, qw, sc, zr, rows)
        y = y[:, rows].astype(np.float64)
    assert np.all(np.isfinite(y)), "non-finite output"
    err = np.abs(y - y_ref)
    lim = RTOL * B + ATOL
    worst = np.unravel_index(np.argmax(err - lim), err.shape)
    assert np.all(err <= lim), f"max excess at {worst}: |{y[worst]} - {y_ref[worst]}| > {lim[worst]}"


def case(dev, M, N, K, seed, bits=4, mode=oracle.ASYM, workspace=None):
    W, x = inputs.random_case(seed, N, K, M)
    qo, so, zo = oracle.quantize_pack(W, None, 128, bits, mode)
    args = (to_dev(x, dev), to_dev(qo.view(np.int32), dev), to_dev(so, dev), to_dev(zo, dev))
    y = w4.w4a16_gemm(*args, workspace=workspace)
    torch.cuda.synchronize()
    check(y.cpu().numpy(), x, qo, so, zo)
    return args, (x, qo, so, zo)


@pytest.mark.parametrize("M,N,K", [
    (5, 1, 128),          # one row, one group, MP = 16
    (8, 300, 1024),       # ragged row block (300 = 256 + 44)
    (16, 256, 128),       # one unit per row block
    (16, 1000, 2048),
    (17, 513, 1152),      # MP = 32, odd groups per row
    (32, 64, 8192),       # many CTAs share one row block
    (48, 129, 4096),      # MP = 48
    (64, 256, 11008),     # 86 groups per row
    (64, 2048, 256),
    (64, 300, 22016),     # 172 groups per row
])
def test_tc_small_shapes(dev, M, N, K):
    case(dev, M, N, K, seed=M * 7919 + N)


@pytest.mark.parametrize("M,N,K", [
    (65, 300, 1024),      # MP = 96, ragged row block
    (96, 513, 2048),
    (100, 256, 1152),     # MP = 128, odd groups per row
    (128, 1000, 4096),
    (128, 64, 8192),      # many CTAs share one row block
])
def test_tc_wide_token_tiles(dev, M, N, K):
    case(dev, M, N, K, seed=M * 7919 + N)


@pytest.mark.parametrize("M,N,K", [
    (129, 300, 1024),     # token tile 192
    (150, 1000, 11008),   # token tile 192, up to 22 CTAs share a tile
    (200, 513, 1152),     # token tile 256, odd groups per row (a pair of one group)
    (256, 384, 2048),     # one full chunk of 256
    (257, 300, 1024),     # 256 + 1: the tail runs on the M = 1 GEMV
    (258, 256, 2048),     # 256 + 2: the tail on the whole-row GEMV for M = 2..4
    (300, 256, 4096),     # 256 + 44
    (512, 384, 2048),     # two full chunks
])
def test_tc_large_m_chunks(dev, M, N, K):
    case(dev, M, N, K, seed=M * 7919 + N)


def test_tc_prefill_workload_sampled_rows(dev):
    """M = 512 tokens on the 8192 x 8192 layer; 128 sampled rows checked for every token."""
    (layer,) = inputs.layer_set(inputs.SKINNY)
    rng = np.random.default_rng(512)
    x = inputs.activations(rng, 512, layer.K, layer.outliers)
    qg, sg, zg = w4.awq_quantize_pack(to_dev(layer.W, dev))
    y = w4.w4a16_gemm(to_dev(x, dev), qg, sg, zg)
    torch.cuda.synchronize()
    rows = np.unique(np.concatenate([rng.choice(layer.N, 124, replace=False), [0, 255, 256, layer.N - 1]]))
    qw = qg.cpu().numpy().view(np.uint32)[rows]
    y_ref, B = oracle.gemm_ref(x, oracle.dequant(qw, sg.cpu().numpy()[rows], zg.cpu().numpy()[rows]))
    err = np.abs(y.cpu().numpy()[:, rows].astype(np.float64) - y_ref)
    assert np.all(err <= RTOL * B + ATOL)


def test_tc_whole_row_blocks_written_directly(dev):
    """K = 128: every CTA covers whole row blocks and writes y without the workspace."""
    case(dev, 33, 40960, 128, seed=11)


def test_tc_3bit_symmetric_codes(dev):
    case(dev, 16, 200, 2048, seed=5, bits=3, mode=oracle.SYM)


@pytest.mark.parametrize("M", [16, 32, 64])
def test_tc_skinny_workload_sampled_rows(dev, M):
    """K = N = 8192 quantized on the GPU, the launch the bench times; 256 sampled rows checked."""
    (layer,) = inputs.layer_set(inputs.SKINNY)
    x = layer.x[:M]
    qg, sg, zg = w4.awq_quantize_pack(to_dev(layer.W, dev))
    y = w4.w4a16_gemm(to_dev(x, dev), qg, sg, zg)
    torch.cuda.synchronize()
    rows = np.unique(np.concatenate([np.random.default_rng(M).choice(layer.N, 252, replace=False),
                                     [0, 255, 256, layer.N - 1]]))
    qw = qg.cpu().numpy().view(np.uint32)[rows]
    y_ref, B = oracle.gemm_ref(x, oracle.dequant(qw, sg.cpu().numpy()[rows], zg.cpu().numpy()[rows]))
    err = np.abs(y.cpu().numpy()[:, rows].astype(np.float64) - y_ref)
    assert np.all(err <= RTOL * B + ATOL)
    qo, _, _ = oracle.quantize_pack(layer.W[rows], None, 128, 4, oracle.ASYM)
    assert np.array_equal(qw, qo)


def test_tc_workspace_shared_across_paths(dev):
    """One workspace serves M = 1, 32, 4, 64, 3 in turn; each result is right, and the
    part the CUDA-core GEMV needs zeroed (its M = 4 size) is left zeroed."""
    N, K = 700, 4096
    ws = torch.zeros(w4.gemm_workspace_size(64, N, K), dtype=torch.uint8, device=dev)
    for i, M in enumerate((1, 32, 4, 64, 3)):
        case(dev, M, N, K, seed=100 + i, workspace=ws)
    w4.gemm_check(ws)
    assert int(ws[:w4.gemm_workspace_size(4, N, K)].count_nonzero()) == 0


def test_tc_repeated_calls_identical(dev):
    """Calls repeat on the same inputs and agree with the oracle every time."""
    args, ref = case(dev, 64, 512, 8192, seed=7)
    y1 = w4.w4a16_gemm(*args).cpu().numpy()
    y2 = w4.w4a16_gemm(*args).cpu().numpy()
    check(y1, *ref)
    check(y2, *ref)


@pytest.mark.parametrize("M", [16, 128, 200, 300])
def test_tc_bit_identical_across_calls(dev, M):
    """The partial tiles of shared row tiles are added in CTA order, so y must not
    change by a single bit from call to call.  At 8192 x 8192 every CTA streams
    about 14 units through its rings, which exposes a ring stage overwritten
    while it is still being read (the tolerance of the parity tests can hide it)."""
    (layer,) = inputs.layer_set(inputs.SKINNY)
    rng = np.random.default_rng(M)
    qg, sg, zg = w4.awq_quantize_pack(to_dev(layer.W, dev))
    x = to_dev(inputs.activations(rng, M, layer.K, layer.outliers), dev)
    ws = torch.zeros(w4.gemm_workspace_size(M, layer.N, layer.K), dtype=torch.uint8, device=dev)
    y0 = w4.w4a16_gemm(x, qg, sg, zg, workspace=ws).clone()
    diff = torch.zeros((), dtype=torch.int64, device=dev)
    for _ in range(20):
        diff += (w4.w4a16_gemm(x, qg, sg, zg, workspace=ws) != y0).sum()
    w4.gemm_check(ws)
    assert int(diff) == 0
