"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Packed codes, scales and zeros must be bit-exact.  The GEMV/GEMM output must
satisfy, per element, |y - y_ref| <= 2e-3 * B + 1e-3 with B = sum_k |x * w_hat|
and y_ref the fp64 product with the dequantized weight.
"""
import numpy as np
import pytest
import torch

import oracle
import w4a16_decode_gemv_b200 as w4
from w4a16_decode_gemv_b200 import build, inputs

pytestmark = pytest.mark.gpu

F16 = np.float16
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


def qw_np(t):
    return t.cpu().numpy().view(np.uint32)


def bits16(a):
    return np.asarray(a, dtype=F16).view(np.uint16)


def quantize_both(W, s, bits, mode, dev):
    Wd = to_dev(W, dev)
    sd = None if s is None else to_dev(s, dev)
    qg, sg, zg = w4.awq_quantize_pack(Wd, sd, 128, bits, mode)
    torch.cuda.synchronize()
    qo, so, zo = oracle.quantize_pack(W, s, 128, bits, mode)
    return (qw_np(qg), sg.cpu().numpy(), zg.cpu().numpy()), (qo, so, zo)


def assert_bit_exact(gpu, ora, what=""):
    qg, sg, zg = gpu
    qo, so, zo = ora
    bad = np.flatnonzero((qg != qo).ravel())
    assert bad.size == 0, f"{what}: {bad.size} packed words differ, first at {bad[:5]}"
    assert np.array_equal(bits16(sg), bits16(so)), f"{what}: scales differ"
    assert np.array_equal(bits16(zg), bits16(zo)), f"{what}: zeros differ"


def assert_close(y, x, qw, sc, zr, rows=None):
    if rows is None:
        y_ref, B = oracle.gemm(x, qw, sc, zr)
        y = y.astype(np.float64)
    else:
        y_ref, B = oracle.gemm_rows(x, qw, sc, zr, rows)
        y = y[:, rows].astype(np.float64)
    err = np.abs(y - y_ref)
    lim = RTOL * B + ATOL
    worst = np.unravel_index(np.argmax(err - lim), err.shape)
    assert np.all(np.isfinite(y)), "non-finite output"
    assert np.all(err <= lim), f"max excess at {worst}: |{y[worst]} - {y_ref[worst]}| > {lim[worst]}"


# ---------------------------------------------------------------------------
# awq_act_scale
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("alpha", [0.5, 0.0, 1.0, 0.25])
def test_act_scale_matches_oracle(dev, alpha):
    _, X, _ = inputs.quant_workload()
    s_gpu = w4.awq_act_scale(to_dev(X, dev), alpha).cpu().numpy()
    s_ora = oracle.act_scale(X, alpha)
    ulps = np.abs(bits16(s_gpu).astype(np.int32) - bits16(s_ora).astype(np.int32))
    # the fp64 sums are exact; pow may differ from libm's by an fp64 ulp, which can
    # move the fp16 result by one ulp only next to a rounding boundary
    assert ulps.max() <= 1
    assert (ulps > 0).sum() <= 2


def test_act_scale_ragged(dev):
    rng = np.random.default_rng(3)
    X = rng.standard_normal((37, 131)).astype(F16)
    s_gpu = w4.awq_act_scale(to_dev(X, dev), 0.5).cpu().numpy()
    assert np.abs(bits16(s_gpu).astype(int) - bits16(oracle.act_scale(X, 0.5)).astype(int)).max() <= 1


# ---------------------------------------------------------------------------
# awq_quantize_pack: bit-exact
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("bits,mode", [(4, w4.ASYM), (3, w4.SYM), (4, w4.SYM), (3, w4.ASYM)])
@pytest.mark.parametrize("N,K", [(1, 128), (3, 256), (17, 1152), (100, 4096), (33, 11008)])
def test_quantize_small_shapes(dev, bits, mode, N, K):
    W, _ = inputs.random_case(N + K, N, K)
    assert_bit_exact(*quantize_both(W, None, bits, mode, dev), f"{N}x{K}")


@pytest.mark.parametrize("bits,mode", [(4, w4.ASYM), (3, w4.SYM)])
def test_quantize_awq_workload_full(dev, bits, mode):
    """11008 x 4096 weight, s = s_X^0.5 from 512 calibration tokens (bit-exact)."""
    W, X, _ = inputs.quant_workload()
    s = oracle.act_scale(X, 0.5)
    assert_bit_exact(*quantize_both(W, s, bits, mode, dev), "11008x4096 awq")


def test_quantize_random_scales(dev):
    rng = np.random.default_rng(7)
    W, _ = inputs.random_case(9, 64, 2048)
    s = np.exp(rng.uniform(-3, 3, size=2048)).astype(F16)
    for bits, mode in [(4, w4.ASYM), (3, w4.SYM)]:
        assert_bit_exact(*quantize_both(W, s, bits, mode, dev), "random s")


def _edge_groups():
    rng = np.random.default_rng(17)
    G = []
    G.append(np.zeros(128))                                   # all zero
    G.append(np.full(128, 0.5))                               # constant positive
    G.append(np.full(128, -3.25))                             # constant negative
    G.append(-np.abs(rng.standard_normal(128)) - 0.1)         # all negative
    G.append(np.abs(rng.standard_normal(128)) + 0.1)          # all positive
    G.append(rng.standard_normal(128) * 1e-6)                 # subnormal fp16 range
    g = np.zeros(128); g[5] = 2.0 ** -24; G.append(g)         # step underflows
    G.append(rng.uniform(-60000, 60000, 128))                 # near the fp16 limit
    g = np.zeros(128); g[0] = -0.0; g[1] = 0.0; G.append(g)   # signed zeros
    # exact ties: step 0.25, elements on half steps
    G.append(np.concatenate([[-0.625, 3.125], (np.arange(126) % 15 - 2) * 0.25 + 0.125]))
    G.append(np.concatenate([[-0.75, 3.0], (np.arange(126) % 14 - 3) * 0.25 + 0.125]))
    G.append(np.concatenate([[-2.0, 2.0], np.linspace(-2, 2, 126)]))
    # max and min so far apart in magnitude that max - min is inexact in fp32
    # (the step then comes from the fp64 path)
    G.append(np.concatenate([[1000.0, -2.0 ** -20], rng.standard_normal(126) * 1e-3]))
    G.append(np.concatenate([[2.0 ** -24, 1000.0], rng.uniform(2.0 ** -24, 1000.0, 126)]))
    return np.stack(G).astype(F16)


@pytest.mark.parametrize("bits,mode", [(4, w4.ASYM), (3, w4.ASYM), (4, w4.SYM), (3, w4.SYM)])
def test_quantize_edge_groups(dev, bits, mode):
    G = _edge_groups()
    W = G.reshape(-1, 256) if G.shape[0] % 2 == 0 else G
    assert_bit_exact(*quantize_both(W, None, bits, mode, dev), "edge groups")
    # AWQ scale that hits exact fp16 product ties; the near-65504 group is left
    # out because W * 1.5 would overflow fp16 (outside the stated precondition)
    G2 = np.delete(G, 7, axis=0)
    W2 = G2.reshape(-1, 256) if G2.shape[0] % 2 == 0 else G2
    s = np.full(W2.shape[1], 1.5, dtype=F16)
    assert_bit_exact(*quantize_both(W2, s, bits, mode, dev), "edge groups, s=1.5")


def _sweep_weight():
    """Every finite fp16 value, placed in groups whose two anchors fix the step."""
    allv = np.arange(0, 1 << 16, dtype=np.uint32).astype(np.uint16).view(F16)
    allv = allv[np.isfinite(allv)].astype(np.float64)
    rows = []

    def add(lo, hi, vals):
        for start in range(0, len(vals), 126):
            g = np.zeros(128)
            g[0], g[1] = lo, hi
            chunk = vals[start:start + 126]
            g[2:2 + len(chunk)] = chunk
            rows.append(g)

    for e in range(-24, 15):
        lo, hi = float(F16(-1.5 * 2.0 ** e)), float(F16(2.0 ** (e + 1)))
        add(lo, hi, allv[(allv >= lo) & (allv <= hi)])
    add(-65504.0, 65504.0, allv[np.abs(allv) >= 2.0 ** 14])   # top binades, widest anchors
    W = np.stack(rows)
    covered = np.unique(W.astype(F16).view(np.uint16))
    assert np.isin(allv.astype(F16).view(np.uint16), covered).all()
    if W.shape[0] % 2:
        W = np.vstack([W, np.zeros((1, 128))])
    return W.reshape(-1, 256).astype(F16)


@pytest.mark.parametrize("bits,mode", [(4, w4.ASYM), (3, w4.ASYM), (4, w4.SYM), (3, w4.SYM)])
def test_quantize_exhaustive_fp16_sweep(dev, bits, mode):
    W = _sweep_weight()
    assert_bit_exact(*quantize_both(W, None, bits, mode, dev), "fp16 sweep")


# ---------------------------------------------------------------------------
# w4a16_gemm (M < 16: CUDA-core split-K GEMV)
# ---------------------------------------------------------------------------
def _gemm_case(dev, M, N, K, seed, bits=4, mode=w4.ASYM, rows=None):
    W, x = inputs.random_case(seed, N, K, M)
    qo, so, zo = oracle.quantize_pack(W, None, 128, bits, mode)
    y = w4.w4a16_gemm(to_dev(x, dev), to_dev(qo.view(np.int32), dev), to_dev(so, dev), to_dev(zo, dev))
    torch.cuda.synchronize()
    assert_close(y.cpu().numpy(), x, qo, so, zo, rows)


@pytest.mark.parametrize("M,N,K", [
    (1, 1, 128), (1, 3, 256), (1, 5, 1152), (1, 17, 4096), (1, 250, 1024),
    (2, 100, 1024), (3, 37, 2048), (4, 64, 8192), (2, 7, 11008), (4, 9, 22016),
])
def test_gemv_small_shapes(dev, M, N, K):
    _gemm_case(dev, M, N, K, seed=M * 1000 + N)


def test_gemv_3bit_symmetric_codes(dev):
    _gemm_case(dev, 1, 96, 2048, seed=5, bits=3, mode=w4.SYM)


def test_gemv_workload_4096(dev):
    """Single GEMV M=1, K=N=4096, every output element."""
    (layer,) = inputs.layer_set(inputs.GEMV_4096)
    qo, so, zo = oracle.quantize_pack(layer.W, None, 128, 4, oracle.ASYM)
    y = w4.w4a16_gemm(to_dev(layer.x, dev), to_dev(qo.view(np.int32), dev), to_dev(so, dev), to_dev(zo, dev))
    torch.cuda.synchronize()
    assert_close(y.cpu().numpy(), layer.x, qo, so, zo)


@pytest.mark.parametrize("spec,name", [
    (inputs.LLAMA65B, "attn_8192x8192"), (inputs.LLAMA65B, "up_22016x8192"),
    (inputs.LLAMA65B, "down_8192x22016"), (inputs.LLAMA7B, "down_proj"), (inputs.LLAMA7B, "gate_proj"),
])
def test_gemv_full_size_sampled_rows(dev, spec, name):
    """Full-size layers quantized on the GPU; 384 sampled output rows checked."""
    (layer,) = inputs.layer_set(spec, only=name)
    qg, sg, zg = w4.awq_quantize_pack(to_dev(layer.W, dev))
    y = w4.w4a16_gemm(to_dev(layer.x, dev), qg, sg, zg)
    torch.cuda.synchronize()
    rng = np.random.default_rng(0)
    rows = np.unique(np.concatenate([rng.choice(layer.N, 380, replace=False), [0, 1, layer.N - 2, layer.N - 1]]))
    qw = qw_np(qg)[rows]
    y_ref, B = oracle.gemm_ref(layer.x, oracle.dequant(qw, sg.cpu().numpy()[rows], zg.cpu().numpy()[rows]))
    err = np.abs(y.cpu().numpy()[:, rows].astype(np.float64) - y_ref)
    assert np.all(err <= RTOL * B + ATOL)
    # the GPU quantizer agrees with the oracle on the sampled rows
    qo, so, zo = oracle.quantize_pack(layer.W[rows], None, 128, 4, oracle.ASYM)
    assert np.array_equal(qw, qo)


def test_gemv_skinny_m4(dev):
    (layer,) = inputs.layer_set(inputs.SKINNY)
    x = layer.x[:4]
    qg, sg, zg = w4.awq_quantize_pack(to_dev(layer.W, dev))
    y = w4.w4a16_gemm(to_dev(x, dev), qg, sg, zg)
    torch.cuda.synchronize()
    rows = np.random.default_rng(1).choice(layer.N, 256, replace=False)
    y_ref, B = oracle.gemm_ref(x, oracle.dequant(qw_np(qg)[rows], sg.cpu().numpy()[rows], zg.cpu().numpy()[rows]))
    assert np.all(np.abs(y.cpu().numpy()[:, rows].astype(np.float64) - y_ref) <= RTOL * B + ATOL)


# w4a16_gemm, M = 2..8 with K a multiple of 256: register-sourced MMAs (gemv_mma.cu)
@pytest.mark.parametrize("M,N,K", [
    (2, 1, 256),        # one row, one unit per row (15 of 16 warps idle)
    (3, 17, 1280),      # ragged 16-row block, 5 units per row
    (5, 300, 4096),
    (8, 1000, 2048),    # every token column of the MMA used
    (6, 33, 8192),
    (2, 64, 11008),     # 43 units per row: warps with 2 and 3 units
    (7, 129, 512),
])
def test_gemv_mma_shapes(dev, M, N, K):
    _gemm_case(dev, M, N, K, seed=M * 7717 + N)


def test_gemv_mma_edge_values(dev):
    """Zero points 0 and 15, steps from tiny to large, outlier activations, rows past
    a 16-row block; every output checked."""
    rng = np.random.default_rng(3)
    N, K, M = 37, 1024, 4
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float16)
    W[0] = np.abs(W[0])                      # a row of one sign: z = 0
    W[1] = -np.abs(W[1])                     # z = 15
    W[2] *= np.float16(1e-3)                 # tiny steps
    W[3] = (rng.standard_normal(K) * 2).astype(np.float16)  # large steps
    x = rng.standard_normal((M, K)).astype(np.float16)
    x[:, :11] *= np.float16(40)              # outlier channels
    qo, so, zo = oracle.quantize_pack(W, None, 128, 4, oracle.ASYM)
    y = w4.w4a16_gemm(to_dev(x, dev), to_dev(qo.view(np.int32), dev), to_dev(so, dev), to_dev(zo, dev))
    torch.cuda.synchronize()
    assert_close(y.cpu().numpy(), x, qo, so, zo)


@pytest.mark.parametrize("M", [2, 4, 8])
def test_gemv_mma_workload_rows_and_repeats(dev, M):
    """The K = N = 8192 skinny layer at M = 2, 4, 8 (the bench's launches): sampled rows
    against the oracle, and y bit-identical over repeated calls."""
    (layer,) = inputs.layer_set(inputs.SKINNY)
    x = layer.x[:M]
    qg, sg, zg = w4.awq_quantize_pack(to_dev(layer.W, dev))
    xd = to_dev(x, dev)
    ys = [w4.w4a16_gemm(xd, qg, sg, zg).cpu().numpy() for _ in range(4)]
    for yy in ys[1:]:
        assert np.array_equal(yy.view(np.uint16), ys[0].view(np.uint16))
    rows = np.unique(np.concatenate([np.random.default_rng(M).choice(layer.N, 250, replace=False),
                                     [0, 15, 16, layer.N - 1]]))
    y_ref, B = oracle.gemm_ref(x, oracle.dequant(qw_np(qg)[rows], sg.cpu().numpy()[rows], zg.cpu().numpy()[rows]))
    assert np.all(np.abs(ys[0][:, rows].astype(np.float64) - y_ref) <= RTOL * B + ATOL)


@pytest.mark.parametrize("M,N,K", [(4, 2048, 22016), (3, 513, 1152), (1, 300, 1152), (2, 512, 65536)])
def test_split_k_gemv_repeats_bit_for_bit(dev, M, N, K):
    """The split-K GEMV (activations too large to stage, or K / 128 odd) adds at most
    two partial sums per output onto zero, so y is the same on every call."""
    W, x = inputs.random_case(M * 13 + N, N, K, M)
    qo, so, zo = oracle.quantize_pack(W[:64], None, 128, 4, oracle.ASYM)
    qg, sg, zg = w4.awq_quantize_pack(to_dev(W, dev))
    assert np.array_equal(qw_np(qg)[:64], qo)
    xd = to_dev(x, dev)
    ys = [w4.w4a16_gemm(xd, qg, sg, zg).cpu().numpy().view(np.uint16) for _ in range(6)]
    for y in ys[1:]:
        assert np.array_equal(y, ys[0])
    y_ref, B = oracle.gemm(x, qo, so, zo)
    err = np.abs(ys[0].view(np.float16)[:, :64].astype(np.float64) - y_ref)
    assert np.all(err <= RTOL * B + ATOL)


def test_workspace_left_zeroed_and_calls_repeat(dev):
    W, x = inputs.random_case(42, 300, 4096, 1)
    qo, so, zo = oracle.quantize_pack(W, None, 128, 4, oracle.ASYM)
    args = [to_dev(x, dev), to_dev(qo.view(np.int32), dev), to_dev(so, dev), to_dev(zo, dev)]
    ws = torch.zeros(w4.gemm_workspace_size(1, 300, 4096), dtype=torch.uint8, device=dev)
    ys = [w4.w4a16_gemm(*args, workspace=ws).cpu().numpy() for _ in range(3)]
    w4.gemm_check(ws)
    assert int(ws.count_nonzero()) == 0
    for y in ys:
        assert_close(y, x, qo, so, zo)
