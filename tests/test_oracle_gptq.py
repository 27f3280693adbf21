"""Pins of the oracle's GPTQ (CPU only).

GPTQ ("CMU 11-868 LLM Systems: Model Quantization" reading guide, §L20 "GPTQ";
"Learning-ML-DL ch. 11", §11.4) quantizes one column at a time and pushes each
column's rounding error onto the columns not yet quantized, through the upper
Cholesky factor G of (2 X^T X + lambda I)^-1.  None of the checks below retypes
that recursion:

* the Hessian against explicit loops over tokens;
* the factor by its defining properties (triangular, positive diagonal,
  G^T G inverts H, checked through a linear solve);
* an identity Hessian, where no error moves and GPTQ is plain RTN;
* the optimal-brain-surgeon property the recursion exists to realise: when
  column i is quantized, the not-yet-quantized columns equal the exact
  minimiser of the output error (w - v)^T H (w - v) given the columns already
  fixed, computed here by solving the linear system directly;
* the qualitative claim of [ML11] §11.4: the weight error goes up, the output
  error goes down, relative to RTN.
"""
import math

import numpy as np
import pytest

import oracle

F16, F64 = np.float16, np.float64


def _rand_w(rng, n, k, sigma=0.02):
    return (rng.standard_normal((n, k)) * sigma).astype(F16)


def _correlated_x(rng, t, k, mix=0.8):
    """Calibration tokens whose channels are correlated (a random mixing of
    independent channels), so that H has large off-diagonal entries."""
    z = rng.standard_normal((t, k))
    a = np.eye(k) + mix * rng.standard_normal((k, k)) / math.sqrt(k)
    return (z @ a).astype(F16)


def test_hessian_matches_token_loops():
    rng = np.random.default_rng(1)
    X = rng.standard_normal((5, 4)).astype(F16)
    T, K = X.shape
    H0 = [[2.0 * math.fsum(float(X[t, i]) * float(X[t, j]) for t in range(T)) for j in range(K)] for i in range(K)]
    lam = 0.01 * math.fsum(H0[i][i] for i in range(K)) / K
    want = np.array(H0) + lam * np.eye(K)
    np.testing.assert_allclose(oracle.gptq_hessian(X), want, rtol=1e-13, atol=0)


def test_factor_is_the_upper_cholesky_factor_of_the_inverse():
    rng = np.random.default_rng(2)
    H = oracle.gptq_hessian(_correlated_x(rng, 64, 12))
    G = oracle.gptq_factor(H)
    assert np.array_equal(G, np.triu(G)), "G must be upper triangular"
    assert np.all(np.diag(G) > 0)
    # G^T G = H^-1  <=>  H (G^T G) = I; compared with a solve, not an inverse
    np.testing.assert_allclose(G.T @ G, np.linalg.solve(H, np.eye(12)), rtol=1e-9, atol=1e-12)
    np.testing.assert_allclose(H @ (G.T @ G), np.eye(12), atol=1e-9)


@pytest.mark.parametrize("bits,mode", [(4, oracle.ASYM), (3, oracle.SYM), (4, oracle.SYM)])
def test_identity_hessian_is_plain_rtn(bits, mode):
    """X = 2 I gives H = c I: G is diagonal, no error reaches another column, and
    the codes, steps and zero points are the RTN ones, bit for bit."""
    rng = np.random.default_rng(3)
    K = 256
    W = _rand_w(rng, 24, K)
    W[0, :128] = F16(0.01)          # a constant group: the zero-range rule
    W[1, 128:] = F16(0.0)
    X = (2.0 * np.eye(K)).astype(F16)
    q, d, z = oracle.gptq_quantize(W, X, 128, bits, mode)
    q0, d0, z0 = oracle.quantize_pack(W, None, 128, bits, mode)
    assert np.array_equal(q, q0)
    assert np.array_equal(d.view(np.uint16), d0.view(np.uint16))
    assert np.array_equal(z.view(np.uint16), z0.view(np.uint16))


@pytest.mark.parametrize("group,bits", [(4, 2), (6, 3), (12, 4)])
def test_each_column_is_the_output_error_minimiser(group, bits):
    """When column i is quantized, columns i.. hold v = w + H[i:, i:]^-1 H[i:, :i] (w - q)[:i]:
    the minimiser over v of (w - u)^T H (w - u) with u = (q[:i], v), solved directly."""
    rng = np.random.default_rng(group * 10 + bits)
    N, K = 3, 12
    W = _rand_w(rng, N, K, sigma=1.0)
    H = oracle.gptq_hessian(_correlated_x(rng, 40, K))
    G = oracle.gptq_factor(H)
    u, d, z, wq = oracle.gptq_sweep(W, G, group, bits, oracle.ASYM)
    d_full = np.repeat(d.astype(F64), group, axis=1)
    z_full = np.repeat(z.astype(F64), group, axis=1)
    q = (u.astype(F64) - z_full) * d_full
    w0 = W.astype(F64)
    for r in range(N):
        for i in range(1, K):
            v = w0[r, i:] + np.linalg.solve(H[i:, i:], H[i:, :i] @ (w0[r, :i] - q[r, :i]))
            assert wq[r, i] == pytest.approx(v[0], rel=1e-9, abs=1e-12), (r, i)
    assert np.array_equal(wq[:, 0], w0[:, 0])


def test_codes_round_the_swept_values():
    """Each code is the RTN code of the value the sweep holds for it, under its group's step."""
    rng = np.random.default_rng(7)
    W = _rand_w(rng, 8, 256)
    G = oracle.gptq_factor(oracle.gptq_hessian(_correlated_x(rng, 300, 256)))
    u, d, z, wq = oracle.gptq_sweep(W, G, 128, 4, oracle.ASYM)
    for r in range(8):
        for i in (0, 1, 127, 128, 200, 255):
            g = i // 128
            dv, zv = float(d[r, g]), float(z[r, g])
            want = min(max(round(wq[r, i] / dv) + zv, 0), 15)   # Python round: half to even
            assert u[r, i] == want


def test_gptq_trades_weight_error_for_output_error():
    """[ML11] §11.4: relative to RTN, GPTQ's weight error is larger and its output
    error ||(W - W_hat) X^T|| smaller (a qualitative check, not the page's ratios)."""
    rng = np.random.default_rng(11)
    K = 256
    W = _rand_w(rng, 48, K)
    X = _correlated_x(rng, 512, K, mix=1.5)
    qg, dg, zg = oracle.gptq_quantize(W, X)
    qr, dr, zr = oracle.quantize_pack(W, None)
    w0 = W.astype(F64)
    e_g = w0 - oracle.dequant(qg, dg, zg)
    e_r = w0 - oracle.dequant(qr, dr, zr)
    xf = X.astype(F64)
    assert np.sum(e_g ** 2) > np.sum(e_r ** 2)
    assert np.sum((e_g @ xf.T) ** 2) < 0.8 * np.sum((e_r @ xf.T) ** 2)


def test_output_is_layout_v1_for_the_gemv():
    """The packed result round-trips through the layout-v1 unpacker and dequantizes
    within half a step of the swept values (codes inside the range)."""
    rng = np.random.default_rng(13)
    W = _rand_w(rng, 16, 256)
    X = _correlated_x(rng, 200, 256)
    G = oracle.gptq_factor(oracle.gptq_hessian(X))
    u, d, z, wq = oracle.gptq_sweep(W, G)
    q, d2, z2 = oracle.gptq_quantize(W, X)
    assert np.array_equal(oracle.unpack_v1(q), u)
    w_hat = oracle.dequant(q, d2, z2)
    step = np.repeat(d2.astype(F64), 128, axis=1)
    inside = (u > 0) & (u < 15)
    assert np.all(np.abs(wq - w_hat)[inside] <= 0.5 * step[inside] * (1 + 1e-12))


def test_group_steps_come_from_the_swept_block():
    """Reading 11: a group's step and zero point are those of its columns as the sweep
    reaches the group, i.e. the output-error minimiser given the earlier groups' codes
    (closed form by a direct solve), not those of the original weights."""
    rng = np.random.default_rng(17)
    N, K, group = 6, 16, 8
    W = _rand_w(rng, N, K, sigma=1.0)
    H = oracle.gptq_hessian(_correlated_x(rng, 40, K, mix=2.0))
    u, d, z, _ = oracle.gptq_sweep(W, oracle.gptq_factor(H), group, 3, oracle.ASYM)
    q0 = (u[:, :group].astype(F64) - z[:, :1].astype(F64)) * d[:, :1].astype(F64)
    w0 = W.astype(F64)
    v = w0[:, group:] + np.linalg.solve(H[group:, group:], H[group:, :group] @ (w0[:, :group] - q0).T).T
    d1, z1 = oracle.group_params(v, 3, oracle.ASYM, group)
    assert np.array_equal(d[:, 1], d1[:, 0]) and np.array_equal(z[:, 1], z1[:, 0])
    d_orig, _ = oracle.group_params(w0[:, group:], 3, oracle.ASYM, group)
    assert not np.array_equal(d[:, 1], d_orig[:, 0]), "the case must tell the two readings apart"


def test_reversed_factorization_gives_the_same_factor():
    """The construction the GPU uses: with P the reversal of the index order, P H P = L L^T and
    G = P L^-1 P is upper triangular with a positive diagonal and G^T G = H^-1, so it equals
    Cholesky(H^-1)^T (uniqueness); no inverse of H is formed."""
    rng = np.random.default_rng(19)
    K = 48
    H = oracle.gptq_hessian(_correlated_x(rng, 80, K, mix=1.5))
    P = np.eye(K)[::-1]
    L = np.linalg.cholesky(P @ H @ P)
    G = P @ np.linalg.solve(L, np.eye(K)) @ P
    assert np.allclose(G, np.triu(G), atol=0) and np.all(np.diag(G) > 0)
    np.testing.assert_allclose(G, oracle.gptq_factor(H), rtol=1e-9, atol=1e-12 * np.abs(G).max())
