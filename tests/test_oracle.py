"""Pins of the CPU oracle against what the pages and the mathematics fix.

No GPU is used.  Each test targets a mistake that could plausibly hide in the
oracle (a dropped term, a wrong sign, index or axis, a wrong denominator,
a wrong rounding mode) and checks it against something other than the
oracle's own formulas: hand-derived values, brute force, invariants the
pages state, or a special case that reduces to a routine the pages print.
"""
import json
import math
import os

import numpy as np
import pytest

import oracle
from oracle import ASYM, SYM

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_groups.json")
F16 = np.float16


def _golden():
    with open(GOLDEN) as f:
        return json.load(f)


def _group_from_case(case):
    g = np.full(128, case["fill"], dtype=np.float64)
    for k, v in case["entries"].items():
        g[int(k)] = v
    g16 = g.astype(F16)
    assert np.array_equal(g16.astype(np.float64), g), "fixture values must be exact fp16"
    return g16[None, :]


# ---------------------------------------------------------------------------
# Hand-derived examples (tests/golden/hand_groups.json)
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("case", _golden()["cases"], ids=lambda c: c["name"])
def test_hand_groups(case):
    wp = _group_from_case(case)
    mode = ASYM if case["mode"] == "asym" else SYM
    d, z = oracle.group_params(wp, case["bits"], mode)
    assert float(d[0, 0]) == case["step"]
    assert float(z[0, 0]) == case["zero"]
    u = oracle.quantize_codes(wp, d, z, case["bits"])[0]
    want = np.full(128, case["fill_code"])
    for k, c in case["codes"].items():
        want[int(k)] = c
    assert np.array_equal(u, want)
    # the packed path gives the same scales/zeros/codes
    qw, sc, zr = oracle.quantize_pack(wp, None, 128, case["bits"], mode)
    assert np.array_equal(oracle.unpack_v1(qw)[0], want)
    assert float(sc[0, 0]) == case["step"] and float(zr[0, 0]) == case["zero"]


@pytest.mark.parametrize("case", _golden()["scaled_weight"]["cases"], ids=lambda c: str(c["s"]))
def test_scaled_weight_single_rounding(case):
    W = np.full((1, 8), case["W"], dtype=F16)
    s = np.full(8, case["s"], dtype=F16)
    assert float(oracle.scale_weight(W, s)[0, 0]) == case["wp"]


def test_act_scale_hand_example():
    g = _golden()["act_scale"]
    X = np.array(g["X"], dtype=F16)
    for alpha, want in g["alphas"].items():
        s = oracle.act_scale(X, float(alpha))
        assert s.dtype == F16 and s.shape == (3,)
        assert [float(v) for v in s] == want, alpha


def test_act_scale_axis_is_tokens():
    # T != K: averaging over the wrong axis changes shape and values
    rng = np.random.default_rng(5)
    X = rng.standard_normal((7, 3)).astype(F16)
    s = oracle.act_scale(X, 1.0)
    assert s.shape == (3,)
    for k in range(3):
        exact = math.fsum(abs(float(v)) for v in X[:, k]) / 7
        assert float(s[k]) == float(F16(exact))


# ---------------------------------------------------------------------------
# Brute force: each code is the nearest representable level
# ---------------------------------------------------------------------------
def _brute_codes(w, d, z, bits):
    """argmin over every code c of |w - (c - z) d|, exact in fp64; ties to even (c - z)."""
    levels = np.arange(2 ** bits, dtype=np.float64)
    out = np.empty(w.shape, dtype=np.int64)
    for idx, wv in np.ndenumerate(w):
        err = np.abs(wv - (levels - z) * d)
        best = np.flatnonzero(err == err.min())
        if len(best) == 2:
            best = [c for c in best if int(c - z) % 2 == 0]
        out[idx] = best[0]
    return out


@pytest.mark.parametrize("bits,mode", [(4, ASYM), (3, ASYM), (4, SYM), (3, SYM)])
@pytest.mark.parametrize("seed", [0, 1, 2])
def test_codes_brute_force_8x128(bits, mode, seed):
    rng = np.random.default_rng(seed)
    W = (rng.standard_normal((8, 128)) * rng.choice([0.02, 1.0, 30.0])).astype(F16)
    if seed == 2:
        # plant exact ties w = (k + 1/2) * step in every row
        d0, _ = oracle.group_params(W, bits, mode)
        for r in range(8):
            W[r, 3] = F16(float(d0[r, 0]) * 1.5)
            W[r, 4] = F16(-float(d0[r, 0]) * 0.5)
    d, z = oracle.group_params(W, bits, mode)
    u = oracle.quantize_codes(W, d, z, bits)
    for r in range(8):
        want = _brute_codes(W[r].astype(np.float64), float(d[r, 0]), float(z[r, 0]), bits)
        assert np.array_equal(u[r], want), r


# ---------------------------------------------------------------------------
# Error invariants: |w - w_hat| <= step/2 except at the clamped edges
# ---------------------------------------------------------------------------
def _roundtrip(W, bits, mode, s=None):
    qw, sc, zr = oracle.quantize_pack(W, s, 128, bits, mode)
    wp = oracle.scale_weight(W, s).astype(np.float64)
    w_hat = oracle.dequant(qw, sc, zr)
    step = np.repeat(sc.astype(np.float64), 128, axis=1)
    return wp, w_hat, step, oracle.unpack_v1(qw)


@pytest.mark.parametrize("bits", [3, 4])
def test_asym_error_bound(bits):
    rng = np.random.default_rng(11)
    W = (rng.standard_normal((64, 1024)) * 0.02).astype(F16)
    wp, w_hat, step, u = _roundtrip(W, bits, ASYM)
    err = np.abs(wp - w_hat)
    top = 2 ** bits - 1
    edge = u == top
    # interior codes: within half a step
    assert np.all(err[~edge] <= step[~edge] / 2)
    # top code may be clamped: the fp16-rounded step can undershoot range/(2^N-1)
    assert np.all(err[edge] <= step[edge] * (0.5 + top * 2.0 ** -11 * 1.01))
    # full code range is used: the group min maps to 0, the max to the top code
    # (or one below it when both halves round down at exact ties)
    g = u.reshape(64, 8, 128)
    assert np.all(g.min(-1) == 0)
    assert np.all(g.max(-1) >= top - 1)
    # and the dequantized range covers the true range to within a step
    wg, hg = wp.reshape(64, 8, 128), w_hat.reshape(64, 8, 128)
    sg = step.reshape(64, 8, 128)[..., 0]
    assert np.all(np.abs(hg.max(-1) - wg.max(-1)) <= sg)
    assert np.all(np.abs(hg.min(-1) - wg.min(-1)) <= sg / 2)


@pytest.mark.parametrize("bits", [3, 4])
def test_sym_error_bound(bits):
    rng = np.random.default_rng(12)
    W = (rng.standard_normal((64, 1024)) * 0.02).astype(F16)
    wp, w_hat, step, u = _roundtrip(W, bits, SYM)
    err = np.abs(wp - w_hat)
    half = 2 ** (bits - 1)
    clamped = wp / step > half - 0.5
    assert np.all(err[~clamped] <= step[~clamped] / 2)
    # positive elements beyond the last level lose up to one step
    assert np.all(err[clamped] <= step[clamped] * (1 + 2.0 ** -10))
    assert np.all(wp[clamped] > 0)
    # the negative extreme is representable: -max|w| maps to code 0
    assert np.all((u == 0) <= (wp < 0))


@pytest.mark.parametrize("mode", [ASYM, SYM])
def test_expected_round_error_quarter_step(mode):
    """Mean |w - w_hat| / step is about 0.25 (Lecture 13 guide, slide 26)."""
    rng = np.random.default_rng(13)
    W = rng.standard_normal((1024, 1024)).astype(F16)  # 1M elements
    wp, w_hat, step, u = _roundtrip(W, 4, mode)
    top = 15
    inner = (u > 0) & (u < top)
    ratio = np.abs(wp - w_hat)[inner] / step[inner]
    assert abs(ratio.mean() - 0.25) < 0.01


# ---------------------------------------------------------------------------
# AWQ: s = 1 is plain RTN; the scaling identity; error shrinks by 1/s
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("bits,mode", [(4, ASYM), (3, SYM)])
def test_unit_scale_is_rtn(bits, mode):
    rng = np.random.default_rng(21)
    W = (rng.standard_normal((16, 512)) * 0.02).astype(F16)
    a = oracle.quantize_pack(W, None, 128, bits, mode)
    b = oracle.quantize_pack(W, np.ones(512, dtype=F16), 128, bits, mode)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)


def test_scaling_identity_exact():
    """(X diag(s)^-1)(W diag(s))^T = X W^T exactly for power-of-two s."""
    rng = np.random.default_rng(22)
    K = 256
    W = (rng.standard_normal((5, K)) * 0.02).astype(F16)
    X = rng.standard_normal((3, K)).astype(F16)
    # s >= 1 keeps every W * s a normal fp16 number, so the product is exact
    s = (2.0 ** rng.integers(0, 4, size=K)).astype(F16)
    s[0] = F16(8.0)  # make the scaled axis unambiguous
    Ws = oracle.scale_weight(W, s)
    Xs = (X.astype(np.float64) / s.astype(np.float64)[None, :])
    y1, _ = oracle.gemm_ref(Xs, Ws.astype(np.float64))
    y0, _ = oracle.gemm_ref(X, W.astype(np.float64))
    assert np.array_equal(y1, y0)
    # scaling rows instead of input channels would break it
    assert not np.array_equal(Ws[:, 0], W[:, 0])


def test_scaling_salient_channel_shrinks_its_error():
    """Scaling channel k by s with the group max unchanged cuts its error ~1/s
    (Lecture 13 guide, AWQ section, slides 26 and 28)."""
    rng = np.random.default_rng(23)
    R, K = 4096, 128
    W = (rng.uniform(-0.5, 0.5, size=(R, K))).astype(F16)
    W[:, 0] = F16(1.0)
    W[:, 1] = F16(-1.0)  # fix max and min of every group
    k0 = 7
    s = np.ones(K, dtype=F16)
    s[k0] = F16(2.0)
    w0 = W[:, k0].astype(np.float64)
    qa = oracle.dequant(*oracle.quantize_pack(W, None, 128, 3, ASYM))[:, k0]
    qb = oracle.dequant(*oracle.quantize_pack(W, s, 128, 3, ASYM))[:, k0] / 2.0
    ea, eb = np.abs(qa - w0).mean(), np.abs(qb - w0).mean()
    assert 0.4 < eb / ea < 0.6


# ---------------------------------------------------------------------------
# Special case: 8-bit asymmetric = the zero-point routine of the CMU guide
# ---------------------------------------------------------------------------
def _zeropoint_int8(X):
    """The zero-point routine described in the CMU 11-868 guide (lecture slide
    10), written here from its description: scale = 255 / range (range 0 -> 1),
    zero point = Round(-scale * min - 128), code = clip(Round(X * scale + zp),
    -128, 127), dequant = (code - zp) / scale."""
    rng_ = X.max() - X.min()
    rng_ = 1.0 if rng_ == 0 else rng_
    scale = 255.0 / rng_
    zp = np.rint(-scale * X.min() - 128)
    q = np.clip(np.rint(X * scale + zp), -128, 127)
    return q, (q - zp) / scale


def test_eight_bit_reduces_to_zero_point_routine():
    rng = np.random.default_rng(31)
    for trial in range(20):
        step = 2.0 ** int(rng.integers(-9, -5))
        lo = -int(rng.integers(1, 254)) * step - step / 4   # z not a tie
        codes = rng.integers(0, 256, size=128).astype(np.float64)
        g = lo + codes * step + rng.uniform(-0.3, 0.3, size=128) * step
        g = np.clip(g, lo, lo + 255 * step)
        g[0], g[1] = lo, lo + 255 * step                     # range = 255 * step
        g = g.astype(F16).astype(np.float64)
        assert g.max() - g.min() == 255 * step
        W = g.astype(F16)[None, :]
        d, z = oracle.group_params(W, 8, ASYM)
        assert float(d[0, 0]) == step
        u = oracle.quantize_codes(W, d, z, 8)[0].astype(np.float64)
        q, deq = _zeropoint_int8(g)
        # the routine rounds w*scale + zp jointly; with an odd zero point the two
        # forms differ only where w/step is an exact half-integer (reading 3)
        tie = (g / step) % 1.0 == 0.5
        assert np.array_equal((u - 128)[~tie], q[~tie])
        w_hat = (u - float(z[0, 0])) * float(d[0, 0])
        assert np.allclose(w_hat[~tie], deq[~tie], rtol=0, atol=1e-12)
        # at ties our code is Round(w/step) + z with Round half to even
        assert np.array_equal(u[tie] - float(z[0, 0]), np.rint(g[tie] / step))


# ---------------------------------------------------------------------------
# Layout v1: pairs come out of one AND with 0x000F000F
# ---------------------------------------------------------------------------
def test_pack_roundtrip_random():
    rng = np.random.default_rng(41)
    u = rng.integers(0, 16, size=(7, 256)).astype(np.uint8)
    qw = oracle.pack_v1(u)
    assert qw.dtype == np.uint32 and qw.shape == (7, 32)
    assert np.array_equal(oracle.unpack_v1(qw), u)


def test_pack_pair_extraction_property():
    """(word >> 4t) & 0x000F000F yields elements (2t, 2t+1) in the low / high halves."""
    rng = np.random.default_rng(42)
    u = rng.integers(0, 16, size=(3, 64)).astype(np.uint8)
    qw = oracle.pack_v1(u)
    for t in range(4):
        pair = (qw >> np.uint32(4 * t)) & np.uint32(0x000F000F)
        assert np.array_equal(pair & 0xFFFF, u[:, 2 * t::8])
        assert np.array_equal(pair >> 16, u[:, 2 * t + 1::8])


@pytest.mark.parametrize("elem", range(8))
def test_pack_single_code_every_slot(elem):
    for v in range(16):
        u = np.zeros((1, 8), dtype=np.uint8)
        u[0, elem] = v
        w = int(oracle.pack_v1(u)[0, 0])
        t, hi = divmod(elem, 2)
        assert (w >> (4 * t + 16 * hi)) & 0xF == v
        assert w & ~(0xF << (4 * t + 16 * hi)) == 0


# ---------------------------------------------------------------------------
# Dequant and the fp64 GEMM against explicit loops
# ---------------------------------------------------------------------------
def test_dequant_and_gemm_loops():
    rng = np.random.default_rng(51)
    M, N, K = 2, 3, 256
    W = (rng.standard_normal((N, K)) * 0.02).astype(F16)
    x = rng.standard_normal((M, K)).astype(F16)
    qw, sc, zr = oracle.quantize_pack(W, None, 128, 4, ASYM)
    u = oracle.unpack_v1(qw)
    w_hat = oracle.dequant(qw, sc, zr)
    for n in range(N):
        for k in range(K):
            g = k // 128
            assert w_hat[n, k] == (float(u[n, k]) - float(zr[n, g])) * float(sc[n, g])
    y, B = oracle.gemm(x, qw, sc, zr)
    assert y.shape == (M, N)
    for m in range(M):
        for n in range(N):
            terms = [float(x[m, k]) * w_hat[n, k] for k in range(K)]
            assert abs(y[m, n] - math.fsum(terms)) <= 1e-12 * math.fsum(abs(t) for t in terms)
            assert abs(B[m, n] - math.fsum(abs(t) for t in terms)) <= 1e-12 * B[m, n]
    yr, Br = oracle.gemm_rows(x, qw, sc, zr, [2, 0])
    assert np.array_equal(yr, y[:, [2, 0]])
